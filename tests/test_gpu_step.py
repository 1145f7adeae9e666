"""lcla_step on the GPU: streaming blocks against the carried state.

The streaming workload (B=2, H=70, 41 latent frames of 30x52 tokens fed as 14
blocks of 3 frames, the last one 2 frames) must reproduce the one-shot
forward and the oracle; save=0 must leave the state bit-unchanged and give
the same outputs every time; a state saved to the host and restored must
continue exactly like an uninterrupted run.
"""
import numpy as np
import pytest
import torch

import block_causal_relu_b200 as lcla
import oracle
from gpu_util import dev, host, inputs_to_dev, sample_rows
from parity import check_outputs, check_state
from workloads import NAMED, Spec, make_inputs

pytestmark = pytest.mark.gpu


def blocks(spec):
    return [(t0, min(spec.N, t0 + spec.block_len)) for t0 in range(0, spec.N, spec.block_len)]


def test_streaming_equals_forward_and_oracle():
    spec = NAMED["stream_bf16"]
    inp = make_inputs(spec)
    q, k, v, c, s = inputs_to_dev(inp)
    full, st_full = lcla.forward(q, k, v, c, s, spec.block_len, spec.eps)
    state = torch.zeros((spec.B, spec.H, 33, 32), device="cuda")
    outs = []
    starts, ends = [], []
    bl = blocks(spec)
    assert len(bl) == 14 and bl[-1][1] - bl[-1][0] == 3120
    for t0, t1 in bl:
        sl = slice(t0, t1)
        qb, kb, vb = (x[:, sl].contiguous() for x in (q, k, v))
        cb, sb = c[sl].contiguous(), s[sl].contiguous()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        o = lcla.step(qb, kb, vb, cb, sb, state, save=True, eps=spec.eps)
        ev1.record()
        outs.append(o)
        starts.append(ev0)
        ends.append(ev1)
    torch.cuda.synchronize()
    stream_out = torch.cat(outs, dim=1)
    # against the one-shot forward (both GPU, both rounded to bf16: one ulp apart at most
    # from rounding alone); each side is held to the half-ulp bar against the oracle
    check_outputs(host(stream_out), host(full), "bf16", "stream vs forward", ulps=1.0)
    check_state(host(state), host(st_full), "stream state vs forward")
    # against the oracle on sampled rows
    rows = sample_rows(spec.N, spec.block_len, 2048, seed=3)
    ref, ref_st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin,
                                       spec.block_len, spec.eps, rows=rows)
    check_outputs(host(stream_out[:, torch.from_numpy(rows).cuda()]), ref, "bf16", "stream vs oracle")
    check_state(host(state), ref_st, "stream state vs oracle")
    ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    print("per-block ms:", " ".join(f"{x:.3f}" for x in ms))


@pytest.mark.parametrize("dtype,L", [("bf16", 4680), ("f32", 1560), ("bf16", 40), ("f32", 1)])
def test_save_flag_semantics(dtype, L):
    spec = Spec("save", 2, 5, 4 * L, 32, L, dtype, 21, qk_dist="laplace_negrows", v_sigma=2.0)
    inp = make_inputs(spec, threads=2)
    q, k, v, c, s = inputs_to_dev(inp)
    rng = np.random.default_rng(1)
    st0 = rng.standard_normal((2, 5, 33, 32)).astype(np.float32)
    st0[:, :, -1, :] = np.abs(st0[:, :, -1, :]) * 50
    state = dev(st0)
    sl = slice(L, 2 * L)
    blk = [x[:, sl].contiguous() for x in (q, k, v)] + [c[sl].contiguous(), s[sl].contiguous()]
    before = state.clone()
    o1 = lcla.step(*blk, state, save=False)
    o2 = lcla.step(*blk, state, save=False)
    torch.cuda.synchronize()
    assert torch.equal(state, before), "save=0 wrote the state"
    assert torch.equal(o1, o2), "repeated save=0 steps differ"
    o3 = lcla.step(*blk, state, save=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o3), "save flag changed the outputs"
    # oracle step from the same carried state
    st64 = st0.astype(np.float64)
    ref = oracle.step(*(np.ascontiguousarray(a[:, sl]) for a in (inp.q, inp.k, inp.v)),
                      inp.rope_cos[sl], inp.rope_sin[sl], st64, save=True, eps=spec.eps)
    check_outputs(host(o3), ref, dtype, f"step {dtype} L={L}")
    check_state(host(state), st64, f"step state {dtype} L={L}")


def test_host_roundtrip_resume():
    """Save the state to the host after a few blocks, restore it into a fresh
    buffer, continue: bit-identical to the uninterrupted stream."""
    spec = Spec("resume", 2, 8, 6 * 1000, 32, 1000, "bf16", 31)
    inp = make_inputs(spec, threads=2)
    q, k, v, c, s = inputs_to_dev(inp)

    def feed(state, rng_blocks):
        outs = []
        for t0, t1 in rng_blocks:
            sl = slice(t0, t1)
            outs.append(lcla.step(q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(),
                                  c[sl].contiguous(), s[sl].contiguous(), state, save=True))
        return outs

    bl = blocks(spec)
    a_state = torch.zeros((2, 8, 33, 32), device="cuda")
    a = feed(a_state, bl)
    b_state = torch.zeros((2, 8, 33, 32), device="cuda")
    b = feed(b_state, bl[:3])
    saved = b_state.cpu().numpy().copy()
    del b_state
    restored = torch.from_numpy(saved).cuda()
    b += feed(restored, bl[3:])
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    assert torch.equal(a_state, restored)


def test_empty_block_is_noop():
    st = torch.randn((1, 2, 33, 32), device="cuda")
    before = st.clone()
    e = torch.empty((1, 0, 2, 32), dtype=torch.bfloat16, device="cuda")
    t = torch.empty((0, 16), device="cuda")
    out = lcla.step(e, e, e, t, t, st, save=True)
    torch.cuda.synchronize()
    assert out.numel() == 0 and torch.equal(st, before)
