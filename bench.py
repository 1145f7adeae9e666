"""Benchmark: block-causal ReLU linear attention forward on B200.

One step = one lcla_forward over the whole workload (pass A partial states,
scan, pass C outputs) with the inputs resident in HBM.  Default workload: the
minute-scale forward, the largest single-GPU workload (B=1, H=70, d=32, 241
frames x 44x80 tokens = 848320 tokens, blocks of 3 frames = 10560 tokens,
bf16, 3D rotary tables); the 480p-like forward (21 frames x 30x52 tokens,
blocks of 4680) is timed beside it and reported under "also".  Prints one
JSON line with the whole-job throughput in attended token-heads per second,
the end-to-end number through the same call with host buffers, the roofline
of the dominant kernel, and the fp64 CPU oracle timed on the host as a
baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-e2e] [--cpu-seconds S] [--parallel replicas|seq]

N > 1 is launched by torchrun (one rank per GPU): by default every rank runs
its own independent copy of the workload (different seed), no data-path
collective; ``--parallel seq`` instead cuts one sequence into runs of whole
blocks, one per rank, with one all-gather of state totals per step.  Timing
is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import NAMED, make_inputs  # noqa: E402

METRIC = "attended tokens*heads/s and achieved HBM GB/s (% of B200 peak), 1 GPU"
UNIT = "token*heads/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="minute_bf16", choices=sorted(NAMED))
    ap.add_argument("--also", default="fwd480p_bf16",
                    help="comma-separated workloads timed after the main one (device time and per-pass "
                         "roofline only), reported under 'also'; 'none' for none")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--parallel", choices=["replicas", "seq"], default="replicas",
                    help="N > 1: replicas = one independent copy of the workload per rank (weak scaling); "
                         "seq = one sequence cut into runs of whole blocks, one per rank, with one "
                         "all-gather of state totals per step (strong scaling)")
    ap.add_argument("--op", choices=["attention", "tconv", "step"], default="attention",
                    help="attention: the block-causal attention forward (the headline); "
                         "tconv: the causal temporal convolution with a cached last frame; "
                         "step: the streaming workload block by block through lcla_step")
    return ap.parse_args()


def workload_config(spec, world):
    cfg = {"workload": f"{spec.name}: B={spec.B} H={spec.H} d={spec.d} N={spec.N} "
                       f"block_len={spec.block_len} ({spec.nblocks} blocks)",
           "B": spec.B, "H": spec.H, "d": spec.d, "N": spec.N, "block_len": spec.block_len,
           "rope": spec.rope if spec.grid is None else f"3d t/h/w 8/12/12 on {spec.grid}",
           "eps": spec.eps, "seed": spec.seed,
           "parallelism": "single GPU" if world == 1 else f"{world} independent replicas (weak)"}
    io = 4 * spec.B * spec.N * spec.H * spec.d * spec.elem_bytes
    cfg["l2"] = (f"inputs larger than L2: {io / 1e6:.0f} MB read+written per step > 126 MB"
                 if io > L2_BYTES else "inputs smaller than L2: L2 flushed between steps")
    return cfg


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# the files the profiled kernels are built from (tensor-core passes, the scans, the temporal convolution);
# the CUDA-core passes in lcla_ffma.cuh and lcla_gen.cuh have no traffic record
KERNEL_SOURCES = ("lcla_common.cuh", "lcla_scan.cuh", "lcla_tc.cuh", "lcla_plan.h", "lcla_tconv.cu")


def source_digest():
    """Digest of the files that define the kernels (ncu counters go stale when they change)."""
    h = hashlib.sha256()
    for f in [os.path.join(ROOT, "block_causal_relu_b200", "csrc", n) for n in KERNEL_SOURCES]:
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, workload):
    """DRAM bytes per launch of ``kernel`` on ``workload`` from the committed
    ncu summary, when it was taken on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("source_digest") != source_digest():
        return None
    ent = rec.get("workloads", {}).get(workload, {}).get(kernel)
    return ent.get("traffic_bytes_per_launch") if ent else None


class ClockSampler:
    """NVML (the library behind nvidia-smi) samples of SM clock, power and
    clock-event reasons on this rank's GPU while running."""
    NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
             0x8: "hw_slowdown", 0x20: "sync_boost", 0x40: "sw_thermal_slowdown",
             0x80: "hw_thermal_slowdown", 0x100: "hw_power_brake_slowdown",
             0x200: "display_clock_setting"}

    def __init__(self, torch_device, period=0.005):
        self.period = period
        self.samples = []
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            idx = torch.cuda._get_nvml_device_index(torch_device)
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that, do not guess
            self.err = repr(e)

    def _one(self):
        nv = self.nv
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                             nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0, int(r)))

    def _loop(self):
        while not self.stop.is_set():
            self._one()
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.stop = threading.Event()
            self._one()
            self.th = threading.Thread(target=self._loop, daemon=True)
            self.th.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop.set()
            self.th.join()
            self._one()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for s in self.samples:
            bits |= s[2]
        reasons = [n for b, n in sorted(self.NAMES.items()) if bits & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples),
                "power_w_max": max(s[1] for s in self.samples), "source": "NVML"}


def head_subset(inp, nh):
    """q, k, v restricted to the first ``nh`` heads (contiguous copies)."""
    sub = lambda a: np.ascontiguousarray(a[:, :, :nh])
    return sub(inp.q), sub(inp.k), sub(inp.v)


def cpu_baseline(inp, seconds):
    """The fp64 oracle (block-recurrence route, every output) on the host cores,
    on a bounded sample: passes over the workload, or over a subset of its
    heads when one whole pass would not fit in ``seconds``, until ``seconds``."""
    import oracle
    orc = oracle.default()
    spec = inp.spec
    threads = orc.max_threads()
    # one pass over as many heads as there are threads (the oracle runs one (b, h) per thread)
    nh = min(spec.H, threads)
    q, k, v = head_subset(inp, nh)
    t0 = time.perf_counter()
    orc.recurrence(q, k, v, inp.rope_cos, inp.rope_sin, spec.block_len, spec.eps)
    per_group = time.perf_counter() - t0
    groups = max(1, int(seconds / 2 / max(per_group, 1e-6)))
    nh = min(spec.H, nh * groups)
    if nh < spec.H:
        q, k, v = head_subset(inp, nh)
    else:
        q, k, v = inp.q, inp.k, inp.v
    n = 0
    t0 = time.perf_counter()
    while True:
        orc.recurrence(q, k, v, inp.rope_cos, inp.rope_sin, spec.block_len, spec.eps)
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds or n >= 50:
            break
    units = spec.B * spec.N * nh
    what = "the whole" if nh == spec.H else f"the first {nh} of {spec.H} heads of the"
    return {"value": n * units / el, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n} pass(es) of the recurrence route over {what} {spec.name} "
                      f"workload ({units} token-heads each, every output and the final "
                      f"state), fp64, {threads} OpenMP threads, {el:.1f} s"}


class Ranks:
    """One process per GPU (torchrun): rank, world size and the two collectives
    the timing needs -- a barrier and the max over ranks of a duration.  The
    data path has none: every rank solves its own problem."""

    def __init__(self, world, rank, backend, device=None, timeout_s=120):
        import torch.distributed as dist
        self.world, self.rank, self.backend, self.device = world, rank, backend, device
        self.dist = dist
        if world > 1:
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)

    def barrier(self):
        if self.world > 1:
            if self.backend == "nccl":
                self.dist.barrier(device_ids=[self.device.index])
            else:
                self.dist.barrier()

    def max(self, x):
        if self.world == 1:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=self.device if self.backend == "nccl" else "cpu")
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            self.dist.destroy_process_group()


def rank_spec(base, rank):
    """Rank r's problem: the same workload with its own seed (independent replicas)."""
    from dataclasses import replace
    return replace(base, seed=base.seed + 1000 * rank)


def whole_job_rate(world, units, steps, ms):
    """Units processed by all ranks per second, timed by the slowest rank (ms over `steps`)."""
    return world * units * steps / (ms / 1e3)


def run_reference(args):
    """Reference arm: the fp64 CPU oracle, rank 0 only, each step a bounded
    sample (a subset of heads) of the same workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    spec = NAMED[args.workload]
    inp = make_inputs(spec)
    orc = oracle.default()
    # calibrate: one pass over as many heads as there are threads (one (b, h) per thread)
    nh = min(spec.H, orc.max_threads())
    q, k, v = head_subset(inp, nh)
    t0 = time.perf_counter()
    orc.recurrence(q, k, v, inp.rope_cos, inp.rope_sin, spec.block_len, spec.eps)
    per_group = max(time.perf_counter() - t0, 1e-4)
    budget = 120.0 / max(1, args.steps + args.warmup)
    nh = int(min(spec.H, nh * max(1, int(budget / per_group))))
    q, k, v = head_subset(inp, nh)
    for _ in range(args.warmup):
        orc.recurrence(q, k, v, inp.rope_cos, inp.rope_sin, spec.block_len, spec.eps)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.recurrence(q, k, v, inp.rope_cos, inp.rope_sin, spec.block_len, spec.eps)
    el = time.perf_counter() - t0
    units = spec.B * spec.N * nh
    val = units * args.steps / el
    line = {"metric": METRIC, "value": val, "unit": UNIT, "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(spec, 1),
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": orc.max_threads(), "kind": "oracle",
                             "sample": f"each step: recurrence route over {nh} of {spec.H} heads "
                                       f"of {spec.name} ({units} token-heads)"},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def e2e_pipelined(device, steps, host_in, dev_in, host_out, dev_out, launch):
    """End-to-end time of ``steps`` steps, each copying its inputs from pinned
    host memory, running the library call and copying its results back, with
    the copies of neighbouring steps overlapped with the compute (PCIe is full
    duplex): step i's uploads run on one stream while step i-1 computes and
    step i-2's results download on a third.  Device inputs and outputs are
    double-buffered (``dev_in[j]``, ``dev_out[j]``, j = step % 2); ``launch(j,
    stream)`` enqueues the step on buffer set j.  Returns ms per step, timed by
    CUDA events from the first upload to the last download."""
    import torch
    s_in, s_cmp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    t0.record(s_in)
    for i in range(steps):
        j = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_cmp[j])          # step i-2 has finished reading buffer set j
            for h, d in zip(host_in, dev_in[j]):
                d.copy_(h, non_blocking=True)
            ev_in[j].record(s_in)
        s_cmp.wait_event(ev_in[j])
        if i >= 2:
            s_cmp.wait_event(ev_out[j])             # step i-2's results have left buffer set j
        launch(j, s_cmp)
        ev_cmp[j].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[j])
            for h, d in zip(host_out, dev_out[j]):
                h.copy_(d, non_blocking=True)
            ev_out[j].record(s_out)
    t1.record(s_out)
    torch.cuda.synchronize(device)
    return t0.elapsed_time(t1) / steps


TCONV = {"name": "tconv480p_bf16", "B": 1, "F": 21, "S": 30 * 52, "C": 2240, "dtype": "bf16", "seed": 11}


def run_tconv(args):
    """One GPU: lcla_temporal_conv over the 480p-like latent (21 frames of
    30 x 52 tokens, width 2240 = 70 heads x 32), with a cached previous frame
    saved each step; inputs resident in HBM and larger than L2.  The JSON line
    keeps the headline's keys with this op's metric."""
    import torch
    import block_causal_relu_b200 as lcla
    from oracle.tconv import temporal_conv as tconv_oracle
    from workloads import f64_to_bf16_bits
    w = TCONV
    B, F, S, C = w["B"], w["F"], w["S"], w["C"]
    rng = np.random.default_rng(w["seed"])
    x_bits = f64_to_bf16_bits(rng.standard_normal(B * F * S * C)).reshape(B, F * S, C)
    c_bits = f64_to_bf16_bits(rng.standard_normal(B * S * C)).reshape(B, S, C)
    wt = rng.standard_normal((2, C)).astype(np.float32)
    bias = rng.standard_normal(C).astype(np.float32)
    dev = torch.device("cuda", 0)
    x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    cache = torch.from_numpy(c_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    wd, bd = torch.from_numpy(wt).to(dev), torch.from_numpy(bias).to(dev)
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream(dev)
    K, W = args.steps, args.warmup
    for _ in range(W):
        lcla.temporal_conv(x, S, wd, bd, cache, save=True, out=y, stream=stream)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        e0.record(stream)
        for _ in range(K):
            lcla.temporal_conv(x, S, wd, bd, cache, save=True, out=y, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / K
    units = B * F * S * C
    bytes_step = 2 * units * 2 + 2 * B * S * C * 2 + 3 * C * 4     # x in, y out, cache in and out, weights
    peak, peak_src = measured_peak()
    achieved = bytes_step / (ms / 1e3) / 1e9
    # end to end: x from pinned host memory, the call, y back (copies overlapped with neighbouring steps)
    xh = x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    KE = max(1, min(args.e2e_steps, K))
    x2, y2 = torch.empty_like(x), torch.empty_like(y)
    xs, ys = [x, x2], [y, y2]
    ems = e2e_pipelined(dev, KE, [xh], [[x], [x2]], [yh], [[y], [y2]],
                        lambda j, st: lcla.temporal_conv(xs[j], S, wd, bd, cache, save=True, out=ys[j], stream=st))
    # the fp64 oracle on the host, same workload, bounded
    n, c0 = 0, time.perf_counter()
    while True:
        tconv_oracle(x_bits, S, wt, bias, c_bits)
        n += 1
        el = time.perf_counter() - c0
        if el >= max(1.0, args.cpu_seconds) or n >= 20:
            break
    line = {"metric": "temporal-conv tokens*channels/s and achieved HBM GB/s, 1 GPU", "op": "tconv",
            "value": units / (ms / 1e3), "unit": "token*channels/s", "n_gpus": 1, "steps": K, "warmup": W,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded)",
            "config": {"workload": f"{w['name']}: B={B} F={F} S={S} C={C}", "cache": "previous frame, saved",
                       "l2": f"x and y {2 * units * 2 / 1e6:.0f} MB per step > 126 MB"},
            "roofline": {"bound": "hbm", "kernel": "temporal_conv_k2", "achieved": achieved, "peak": peak,
                         "peak_source": peak_src, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": ncu_traffic("temporal_conv_k2", w["name"]),
                         "algorithmic_bytes": bytes_step},
            "cpu_baseline": {"value": n * units / el, "unit": "token*channels/s", "cores": 1, "kind": "oracle",
                             "sample": f"{n} whole call(s) of the numpy fp64 oracle, {el:.1f} s"},
            "e2e": {"value": units / (ems / 1e3), "unit": "token*channels/s",
                    "h2d_bytes_per_step": units * 2, "d2h_bytes_per_step": units * 2, "ms_per_step": ems,
                    "steps": KE, "overlap": "step i's upload, step i-1's kernel and step i-2's download "
                                            "run on three streams"},
            "gpu_launches": K, "clocks": clk.summary()}
    print(json.dumps(line), flush=True)


def run_step(args):
    """One GPU: the streaming workload (B=2, H=70, 41 latent frames of 30 x 52
    tokens) fed block by block through lcla_step with save=1 -- 13 blocks of
    4680 tokens and one of 3120 -- against the carried state, the blocks'
    inputs resident in HBM.  A step is the whole 14-block sequence; the line
    reports the mean device time per full block, eager (one call per block,
    events around each) and as a CUDA graph of the whole sequence."""
    import torch
    import block_causal_relu_b200 as lcla
    spec = NAMED["stream_bf16"]
    dev = torch.device("cuda", 0)
    inp = make_inputs(spec)

    def to_dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    L = spec.block_len
    bounds = [(t, min(spec.N, t + L)) for t in range(0, spec.N, L)]
    blocks = [[to_dev(a[:, t0:t1]) for a in (inp.q, inp.k, inp.v)] + [to_dev(inp.rope_cos[t0:t1]),
                                                                      to_dev(inp.rope_sin[t0:t1])]
              for t0, t1 in bounds]
    outs = [torch.empty_like(b[0]) for b in blocks]
    state = torch.zeros((spec.B, spec.H, spec.d + 1, spec.d), dtype=torch.float32, device=dev)
    ws = torch.empty(lcla.step_workspace_bytes(spec.B, spec.H, L, spec.d, lcla.BF16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def sequence(events=None):
        state.zero_()
        for i, b in enumerate(blocks):
            if events is not None:
                events[i][0].record(stream)
            lcla.step(*b, state, True, spec.eps, out=outs[i], workspace=ws, stream=stream)
            if events is not None:
                events[i][1].record(stream)

    K, W = args.steps, args.warmup
    for _ in range(W):
        sequence()
    torch.cuda.synchronize(dev)
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in blocks] for _ in range(K)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        e0.record(stream)
        for r in range(K):
            sequence(evs[r])
        e1.record(stream)
        torch.cuda.synchronize(dev)
    ms_seq = e0.elapsed_time(e1) / K
    full = [i for i, (t0, t1) in enumerate(bounds) if t1 - t0 == L]
    per_block = statistics.mean(evs[r][i][0].elapsed_time(evs[r][i][1]) for r in range(K) for i in full)
    # the same sequence replayed as one CUDA graph
    graph_ms = None
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            sequence()                                   # warm up on the capture stream
        stream.wait_stream(side)
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(g):
            cap = torch.cuda.current_stream(dev)
            state.zero_()
            for i, b in enumerate(blocks):
                lcla.step(*b, state, True, spec.eps, out=outs[i], workspace=ws, stream=cap)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize(dev)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(K):
            g.replay()
        g1.record(stream)
        torch.cuda.synchronize(dev)
        graph_ms = g0.elapsed_time(g1) / K
    except Exception as e:  # report, do not hide: the eager numbers stand on their own
        graph_ms = f"capture failed: {type(e).__name__}: {e}"
    tok_heads = spec.B * spec.N * spec.H
    blk_bytes = 4 * spec.B * L * spec.H * spec.d * 2 + 2 * L * (spec.d // 2) * 4 + 2 * spec.B * spec.H * 33 * 32 * 4
    peak, peak_kind = measured_peak()
    achieved = blk_bytes / (per_block / 1e3) / 1e9
    line = {"metric": "streaming blocks: attended tokens*heads/s and ms per full block, 1 GPU", "op": "step",
            "value": tok_heads / (ms_seq / 1e3), "unit": UNIT, "n_gpus": 1, "steps": K, "warmup": W,
            "ms_per_step": ms_seq, "ms_per_block": per_block,
            "graph_ms_per_step": graph_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded)",
            "config": {"workload": f"{spec.name}: B={spec.B} H={spec.H} N={spec.N}, {len(blocks)} blocks of "
                                   f"{L} tokens (last {bounds[-1][1] - bounds[-1][0]}), save=1 each",
                       "l2": f"a full block moves {blk_bytes / 1e6:.0f} MB"},
            "roofline": {"bound": "hbm", "kernel": "one full block (pass A + scan + pass C)", "achieved": achieved,
                         "peak": peak, "peak_source": f"{peak_kind} hbm_gbs", "unit": "GB/s", "frac": achieved / peak,
                         "traffic": None, "algorithmic_bytes": blk_bytes},
            "cpu_baseline": None, "e2e": None, "gpu_launches": K * len(blocks) * 3, "clocks": clk.summary()}
    print(json.dumps(line), flush=True)


def run_seq(args):
    """Sequence-sharded forward: every rank holds the whole-block run
    ``shard_bounds(N, block_len, world)[rank]`` of one sequence; a step is
    lcla_shard_begin, one NCCL all-gather of the state totals, lcla_shard_end.
    The value counts the sequence's token-heads once (strong scaling)."""
    import torch
    import block_causal_relu_b200 as lcla
    from block_causal_relu_b200.seqshard import gather_totals, shard_bounds

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N>1 with torchrun")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    ranks = Ranks(world, rank, "nccl", device)
    spec = NAMED[args.workload]                                # one sequence, the same on every rank
    inp = make_inputs(spec)
    t0, t1 = shard_bounds(spec.N, spec.block_len, world)[rank]
    Nr = t1 - t0

    def to_dev(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(a).to(device)

    q, k, v = (to_dev(a[:, t0:t1]) for a in (inp.q, inp.k, inp.v))
    c, s = to_dev(inp.rope_cos[t0:t1]), to_dev(inp.rope_sin[t0:t1])
    code = lcla.BF16 if spec.dtype == "bf16" else lcla.F32
    out = torch.empty_like(q)
    st = torch.empty((spec.B, spec.H, spec.d + 1, spec.d), dtype=torch.float32, device=device)
    total = torch.empty_like(st)
    ws = torch.empty(max(1, lcla.shard_workspace_bytes(spec.B, spec.H, Nr, spec.d, spec.block_len, code)),
                     dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        lcla.shard_begin(k, v, c, s, spec.block_len, total_out=total, workspace=ws, stream=stream)
        totals = gather_totals(total)
        lcla.shard_end(q, k, v, c, s, spec.block_len, totals, rank, ws, spec.eps, out=out, state_out=st,
                       stream=stream)

    def barrier():
        ranks.barrier()
        torch.cuda.synchronize(device)

    K, W = args.steps, args.warmup
    for _ in range(W):
        step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device) as clk:
        e0.record(stream)
        for _ in range(K):
            step()
        e1.record(stream)
        torch.cuda.synchronize(device)
    barrier()
    ms_total = ranks.max(e0.elapsed_time(e1))
    ms = ms_total / K
    plan = lcla.plan_info(spec.B, spec.H, max(Nr, 1), spec.d, spec.block_len, code)
    esz = spec.elem_bytes
    local_bytes = 4 * spec.B * Nr * spec.H * spec.d * esz + 2 * 2 * Nr * (spec.d // 2) * 4
    slowest_bytes = ranks.max(float(local_bytes))
    peak, peak_kind = measured_peak()
    achieved = slowest_bytes / (ms / 1e3) / 1e9
    if rank == 0:
        ngroups = plan["segments"] if plan["chunk_mode"] else plan["prefixes"]
        scan_k = 1 if ngroups <= 256 else 2
        cfg = workload_config(spec, world)
        cfg["parallelism"] = (f"sequence sharded over {world} rank(s): whole blocks per rank, "
                              f"one all-gather of {spec.B * spec.H * (spec.d + 1) * spec.d * 4} B per rank per step")
        line = {"metric": METRIC, "value": spec.token_heads / (ms / 1e3), "unit": UNIT, "n_gpus": world,
                "steps": K, "warmup": W, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
                "vs_baseline": None, "dtype": spec.dtype, "data": "synthetic (seeded)", "config": cfg,
                "roofline": {"bound": "hbm", "kernel": "whole sharded step (largest shard)", "achieved": achieved,
                             "peak": peak, "peak_source": f"{peak_kind} hbm_gbs", "unit": "GB/s",
                             "frac": achieved / peak, "traffic": None, "algorithmic_bytes": slowest_bytes},
                "cpu_baseline": None, "e2e": None,
                "gpu_launches": K * (2 + 2 * scan_k + 1), "clocks": clk.summary()}
        print(json.dumps(line), flush=True)
    ranks.close()


def to_dev(a, device):
    """numpy array (bf16 as uint16 bits, or float32) -> torch tensor on ``device``."""
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a).to(device)


def forward_buffers(lcla, spec, device):
    """Device inputs, outputs and workspace of one forward of ``spec``."""
    import torch
    inp = make_inputs(spec)
    ins = tuple(to_dev(a, device) for a in (inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin))
    code = lcla.BF16 if spec.dtype == "bf16" else lcla.F32
    out = torch.empty_like(ins[0])
    st = torch.empty((spec.B, spec.H, spec.d + 1, spec.d), dtype=torch.float32, device=device)
    ws = torch.empty(max(1, lcla.forward_workspace_bytes(spec.B, spec.H, spec.N, spec.d, spec.block_len, code)),
                     dtype=torch.uint8, device=device)
    return inp, ins, out, st, ws


def time_forward(lcla, spec, inputs, out, st, ws, stream, device, K, W, ranks, clocks=False):
    """W warm-up forwards, then two timed regions of K forwards each on
    ``stream``: plain calls back to back (the step time; NVML clocks sampled
    when ``clocks``), then lcla_forward_timed with events between the passes
    (the per-pass times of the roofline; events between the passes would
    defeat the programmatic-launch overlap, so they stay out of the first
    region).  Device times are the max over ranks."""
    import torch
    q, k, v, c, s = inputs
    code = lcla.BF16 if spec.dtype == "bf16" else lcla.F32
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    for row in evs:                       # materialise the event handles
        for e in row:
            e.record(stream)

    def step(events=None):
        lcla.forward(q, k, v, c, s, spec.block_len, spec.eps, out=out, state_out=st,
                     workspace=ws, stream=stream, events=events)

    def barrier():
        ranks.barrier()
        torch.cuda.synchronize(device)

    for _ in range(W):
        step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(device) if clocks else None
    if clk:
        clk.__enter__()
    e0.record(stream)
    for _ in range(K):
        step()
    e1.record(stream)
    torch.cuda.synchronize(device)
    if clk:
        clk.__exit__(None, None, None)
    barrier()
    ms_total = ranks.max(e0.elapsed_time(e1))
    for i in range(K):
        step(evs[i])
    torch.cuda.synchronize(device)
    barrier()
    pa = [r[0].elapsed_time(r[1]) for r in evs]
    sc = [r[1].elapsed_time(r[2]) for r in evs]
    pc = [r[2].elapsed_time(r[3]) for r in evs]
    esz = spec.elem_bytes
    tok_bytes = spec.B * spec.N * spec.H * spec.d * esz             # one [B, N, H, d] tensor
    tab_bytes = 2 * spec.N * (spec.d // 2) * 4
    plan = lcla.plan_info(spec.B, spec.H, spec.N, spec.d, spec.block_len, code)
    nseg, npref = plan["segments"], plan["prefixes"]
    sl = spec.B * spec.H * (spec.d + 1) * spec.d * 4
    bytes_a = 2 * tok_bytes + tab_bytes + nseg * sl
    # chunk mode re-reads k and v in pass C for the in-tile term
    bytes_c = (4 if plan["chunk_mode"] else 2) * tok_bytes + tab_bytes + npref * sl
    bytes_s = nseg * sl + npref * sl + sl
    # the grouped scan serves plans with at most 256 prefix groups (blocks, or segments in chunk mode);
    # larger plans scan in chunks with two kernels, timed together
    scan_name = "scan_states_grouped" if (plan["segments"] if plan["chunk_mode"] else plan["prefixes"]) <= 256 \
        else "scan_chunk_totals+scan_chunk_prefix"
    if plan["tensor_cores"]:
        name_a, name_c = "pass_a_tc", "pass_c_tc"
    elif spec.d != 32:
        name_a, name_c = "pass_a_gen", "pass_c_gen"
    else:
        name_a, name_c = "pass_a_ffma", "pass_c_chunk_ffma" if plan["chunk_mode"] else "pass_c_ffma"
    passes = {"pass_a": (statistics.mean(pa), bytes_a, name_a),
              "scan": (statistics.mean(sc), bytes_s, scan_name),
              "pass_c": (statistics.mean(pc), bytes_c, name_c)}
    dom = max(passes, key=lambda kk: passes[kk][0])
    dms, dbytes, dname = passes[dom]
    peak, peak_kind = measured_peak()
    achieved = dbytes / (dms / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": dname, "achieved": achieved, "peak": peak,
                "peak_source": f"{peak_kind} hbm_gbs", "unit": "GB/s", "frac": achieved / peak,
                "traffic": ncu_traffic(dname, spec.name), "algorithmic_bytes": dbytes}
    path_bytes = 4 * tok_bytes + 2 * tab_bytes + sl      # q,k,v in + out + tables + state
    ms = ms_total / K
    launches = 2 + (1 if scan_name == "scan_states_grouped" else 2)
    return {"ms_per_step": ms, "ms_total": ms_total, "clocks": clk.summary() if clk else None,
            "launches_per_step": launches,
            "pass_ms": {kk: vv[0] for kk, vv in passes.items()},
            "pass_frac_of_peak": {kk: vv[1] / (vv[0] / 1e3) / 1e9 / peak for kk, vv in passes.items()},
            "roofline": roofline, "path_bytes": path_bytes, "tok_bytes": tok_bytes,
            "tab_bytes": tab_bytes, "state_bytes": sl,
            "hbm_frac_of_peak": path_bytes / (ms / 1e3) / 1e9 / peak}


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "tconv":
        return run_tconv(args)
    if args.op == "step":
        return run_step(args)
    if args.parallel == "seq":
        return run_seq(args)

    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N>1 with torchrun")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    ranks = Ranks(world, rank, "nccl", device)

    def barrier():
        ranks.barrier()
        torch.cuda.synchronize(device)

    import block_causal_relu_b200 as lcla

    stream = torch.cuda.current_stream(device)
    K, W = args.steps, args.warmup
    spec = rank_spec(NAMED[args.workload], rank)             # independent problem per rank
    inp, (q, k, v, c, s), out, st, ws = forward_buffers(lcla, spec, device)
    res = time_forward(lcla, spec, (q, k, v, c, s), out, st, ws, stream, device, K, W, ranks, clocks=True)
    ms, ms_total = res["ms_per_step"], res["ms_total"]
    units = spec.token_heads
    value = whole_job_rate(world, units, K, ms_total)
    tok_bytes, tab_bytes, sl = res["tok_bytes"], res["tab_bytes"], res["state_bytes"]

    # end to end through the same call with host buffers
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (torch.empty(q.shape, dtype=q.dtype, pin_memory=True) for _ in range(3))
        hq.copy_(q); hk.copy_(k); hv.copy_(v)
        hc = torch.empty(c.shape, dtype=c.dtype, pin_memory=True); hc.copy_(c)
        hs = torch.empty(s.shape, dtype=s.dtype, pin_memory=True); hs.copy_(s)
        hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        hst = torch.empty(st.shape, dtype=st.dtype, pin_memory=True)
        KE = max(1, min(args.e2e_steps, K))
        ins = [[q, k, v, c, s], [torch.empty_like(t) for t in (q, k, v, c, s)]]
        outs = [[out, st], [torch.empty_like(out), torch.empty_like(st)]]

        def e2e_launch(j, stream_j):
            qq, kk, vv, cc, ss = ins[j]
            lcla.forward(qq, kk, vv, cc, ss, spec.block_len, spec.eps, out=outs[j][0], state_out=outs[j][1],
                         workspace=ws, stream=stream_j)

        e2e_pipelined(device, 2, [hq, hk, hv, hc, hs], ins, [hout, hst], outs, e2e_launch)   # warm the streams
        barrier()
        ems = ranks.max(KE * e2e_pipelined(device, KE, [hq, hk, hv, hc, hs], ins, [hout, hst], outs,
                                           e2e_launch))
        barrier()
        h2d = 3 * tok_bytes + tab_bytes
        d2h = tok_bytes + sl
        e2e = {"value": whole_job_rate(world, units, KE, ems), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": ems / KE, "steps": KE,
               "overlap": "step i's upload, step i-1's forward and step i-2's download run on three streams"}
        del hq, hk, hv, hc, hs, hout, hst, ins, outs

    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        cpu = cpu_baseline(inp, args.cpu_seconds)
    del inp, q, k, v, c, s, out, st, ws
    torch.cuda.empty_cache()

    # the other workloads of --also: device time and per-pass roofline each
    also = {}
    for name in [n for n in args.also.split(",") if n and n != "none" and n != args.workload]:
        aspec = rank_spec(NAMED[name], rank)
        _, ains, aout, ast, aws = forward_buffers(lcla, aspec, device)
        r = time_forward(lcla, aspec, ains, aout, ast, aws, stream, device, K, W, ranks)
        also[name] = {"workload": workload_config(aspec, world)["workload"], "ms_per_step": r["ms_per_step"],
                      "value": whole_job_rate(world, aspec.token_heads, K, r["ms_total"]),
                      "hbm_frac_of_peak": r["hbm_frac_of_peak"], "pass_ms": r["pass_ms"],
                      "pass_frac_of_peak": r["pass_frac_of_peak"], "roofline": r["roofline"]}
        del ains, aout, ast, aws
        torch.cuda.empty_cache()

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
                "warmup": W, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": spec.dtype, "data": "synthetic (seeded)",
                "config": workload_config(spec, world),
                "achieved_hbm_gbs": res["path_bytes"] / (ms / 1e3) / 1e9,
                "hbm_frac_of_peak": res["hbm_frac_of_peak"],
                "pass_ms": res["pass_ms"], "pass_frac_of_peak": res["pass_frac_of_peak"],
                "roofline": res["roofline"], "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": res["launches_per_step"] * K, "clocks": res["clocks"], "also": also}
        print(json.dumps(line), flush=True)
    ranks.close()


if __name__ == "__main__":
    main()
