"""The multi-GPU bench path's host logic, on CPU with two gloo ranks.

bench.py runs one independent replica per rank (the path partitions into
independent (b, h) problems, so there is no data-path collective): each rank
draws its own seeded problem, the timing is the max over ranks, and the
reported value is the whole job's units over that time.  These tests run the
same helpers under two spawned gloo processes; no GPU is involved."""
import importlib.util
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    bench = load_bench()
    from workloads import NAMED, make_inputs
    ranks = bench.Ranks(world, rank, "gloo", timeout_s=60)
    ranks.barrier()
    # the slowest rank decides the time
    t = ranks.max(10.0 * (rank + 1))
    spec = bench.rank_spec(NAMED["tiny_f32"], rank)
    inp = make_inputs(spec, threads=1)
    np.save(os.path.join(out_dir, f"q{rank}.npy"), inp.q)
    with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
        f.write(f"{t} {spec.seed}\n")
    ranks.barrier()
    ranks.close()


@pytest.mark.timeout(240)
def test_two_gloo_ranks_max_and_independent_problems(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [open(tmp_path / f"r{r}.txt").read().split() for r in range(world)]
    assert [float(x[0]) for x in res] == [20.0, 20.0]            # every rank sees the max
    seeds = [int(x[1]) for x in res]
    assert len(set(seeds)) == world                              # one seed per rank
    q0, q1 = (np.load(tmp_path / f"q{r}.npy") for r in range(world))
    assert q0.shape == q1.shape and not np.array_equal(q0, q1)   # independent problems


def test_whole_job_rate_and_single_rank_helpers():
    bench = load_bench()
    # 2 ranks x 1000 units x 10 steps in 5 ms (the slowest rank) -> 4e6 units/s
    assert bench.whole_job_rate(2, 1000, 10, 5.0) == pytest.approx(4e6)
    assert bench.whole_job_rate(1, 1000, 10, 5.0) == pytest.approx(2e6)
    r = bench.Ranks(1, 0, "gloo")        # world 1: no process group, collectives are identities
    assert r.max(3.5) == 3.5
    r.barrier()
    r.close()
    sys.path.insert(0, ROOT)
    from workloads import NAMED
    assert bench.rank_spec(NAMED["fwd480p_bf16"], 0).seed == NAMED["fwd480p_bf16"].seed
    assert bench.rank_spec(NAMED["fwd480p_bf16"], 3).seed == NAMED["fwd480p_bf16"].seed + 3000


def test_reference_arm_non_zero_rank_does_no_work(monkeypatch, capsys):
    """Under torchrun only rank 0 runs (and prints) the CPU reference arm."""
    bench = load_bench()
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"])
    assert bench.run_reference(bench.parse()) is None
    assert capsys.readouterr().out == ""


def test_reference_arm_rank0_prints_the_contract_line(monkeypatch, capsys):
    """Rank 0 times the fp64 oracle on the tiny workload and prints one JSON line
    with the keys the driver reads."""
    import json
    bench = load_bench()
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--workload", "tiny_f32",
                                      "--steps", "2", "--warmup", "1"])
    bench.run_reference(bench.parse())
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_default_workload_is_minute_scale_and_cpu_baseline_takes_a_head_subset(monkeypatch):
    """The headline is the largest single-GPU workload; the CPU baseline of a
    workload too large for its time budget times a labelled subset of heads."""
    bench = load_bench()
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    a = bench.parse()
    assert a.workload == "minute_bf16" and "fwd480p_bf16" in a.also.split(",")
    sys.path.insert(0, ROOT)
    from dataclasses import replace
    from workloads import NAMED, make_inputs
    spec = replace(NAMED["tiny_f32"], H=40, N=4096, block_len=512)
    inp = make_inputs(spec, threads=1)
    cb = bench.cpu_baseline(inp, 1e-9)          # a budget too small for any whole pass
    assert cb["kind"] == "oracle" and cb["value"] > 0
    assert "heads of the" in cb["sample"] and f"of {spec.H} heads" in cb["sample"]
