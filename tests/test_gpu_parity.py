"""lcla_forward on the GPU against the fp64 oracle, element by element.

Small cases that span several tiles, ragged tails and odd head counts are
compared in full against both oracle routes; the robustness sweep (B=1, H=16,
N=65536, block_len in {1, 64, 1560, 4680, N}, fp32 and bf16) is compared in
full against the recurrence route; the 480p-like and minute-scale forwards
run at full size in the launch configuration the benchmark times and are
compared on sampled rows plus the full carried state.
"""
import numpy as np
import pytest
import torch

import block_causal_relu_b200 as lcla
import oracle
from gpu_util import host, inputs_to_dev, sample_rows
from parity import check_outputs, check_state
from workloads import NAMED, Spec, make_inputs

pytestmark = pytest.mark.gpu


def run_gpu(inp, stream=None):
    q, k, v, c, s = inputs_to_dev(inp)
    out, st = lcla.forward(q, k, v, c, s, inp.spec.block_len, inp.spec.eps, stream=stream)
    torch.cuda.synchronize()
    return out, st


SMALL = [  # (B, H, N, block_len, dtype, dist)
    (1, 2, 1000, 64, "f32", "normal"),
    (2, 3, 777, 65, "bf16", "laplace_negrows"),
    (1, 5, 300, 1, "f32", "laplace_negrows"),
    (1, 1, 129, 3, "bf16", "normal"),
    (2, 2, 1500, 100, "f32", "normal"),
    (1, 4, 4096, 4096, "bf16", "normal"),
    (1, 3, 500, 1000, "f32", "normal"),
    (1, 2, 64, 64, "bf16", "normal"),
    (1, 2, 65, 64, "f32", "normal"),
    (1, 2, 63, 64, "bf16", "laplace_negrows"),
    (3, 1, 200, 7, "f32", "normal"),
    (1, 70, 1000, 128, "bf16", "normal"),
    (1, 6, 2000, 33, "f32", "laplace_negrows"),
    (2, 7, 3001, 250, "bf16", "normal"),
    (1, 2, 1, 1, "f32", "normal"),
    (1, 2, 5, 9, "bf16", "normal"),
    # more than 256 blocks: the scan runs in chunks (two kernels)
    (1, 5, 20000, 64, "bf16", "normal"),
    (2, 3, 17000, 64, "f32", "laplace_negrows"),
    (1, 6, 30000, 100, "bf16", "laplace_negrows"),
]


@pytest.mark.parametrize("B,H,N,L,dtype,dist", SMALL)
def test_small_cases_full(B, H, N, L, dtype, dist):
    spec = Spec("small", B, H, N, 32, L, dtype, 1000 + N + L, qk_dist=dist, v_sigma=2.0)
    inp = make_inputs(spec, threads=1)
    out, st = run_gpu(inp)
    ref, ref_st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, L, spec.eps)
    check_outputs(host(out), ref, dtype, f"small {spec}")
    check_state(host(st), ref_st, f"small state {spec}")
    if N * N * H * B <= 4e7:
        msk = oracle.masked(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, L, spec.eps)
        check_outputs(host(out), msk, dtype, f"small vs masked {spec}")


def test_tiny_f32_full():
    spec = NAMED["tiny_f32"]
    inp = make_inputs(spec)
    out, st = run_gpu(inp)
    msk = oracle.masked(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, spec.block_len, spec.eps)
    ref, ref_st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin,
                                       spec.block_len, spec.eps)
    check_outputs(host(out), msk, "f32", "tiny vs masked")
    check_outputs(host(out), ref, "f32", "tiny vs recurrence")
    check_state(host(st), ref_st, "tiny state")


@pytest.mark.parametrize("L", [1, 64, 1560, 4680, 65536])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_robustness_sweep_full(L, dtype):
    spec = NAMED[f"robust_{dtype}_L{L}"]
    inp = make_inputs(spec)
    out, st = run_gpu(inp)
    ref, ref_st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, L, spec.eps)
    o = host(out)
    worst = check_outputs(o, ref, dtype, spec.name)
    check_state(host(st), ref_st, spec.name + " state")
    # rows of q with no positive entry give exact zeros
    qf = inp.as_f32("q")
    zero_rows = (qf <= 0).all(axis=-1)
    assert zero_rows.mean() > 0.25
    assert np.all(o[zero_rows] == 0.0)
    # the pair-by-pair definition on a few rows
    rows = sample_rows(spec.N, L, 24, seed=L)
    msk = oracle.masked(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, L, spec.eps, rows=rows)
    check_outputs(o[:, rows], msk, dtype, spec.name + " vs masked")
    print(f"{spec.name}: worst output excess {worst:.2e}")


@pytest.mark.parametrize("name,nrows", [("fwd480p_bf16", 4096), ("minute_bf16", 1024)])
def test_full_size_sampled(name, nrows):
    spec = NAMED[name]
    inp = make_inputs(spec)
    q, k, v, c, s = inputs_to_dev(inp)
    ws = torch.empty(lcla.forward_workspace_bytes(spec.B, spec.H, spec.N, 32, spec.block_len, 0),
                     dtype=torch.uint8, device="cuda")
    out, st = lcla.forward(q, k, v, c, s, spec.block_len, spec.eps, workspace=ws)
    torch.cuda.synchronize()
    rows = sample_rows(spec.N, spec.block_len, nrows, seed=7)
    ref, ref_st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin,
                                       spec.block_len, spec.eps, rows=rows)
    o = host(out[:, torch.from_numpy(rows).cuda()])
    worst = check_outputs(o, ref, "bf16", name)
    s_err, z_err, fro = check_state(host(st), ref_st, name + " state")
    # the whole output is finite and the same call twice is bit-identical
    assert torch.isfinite(out.float()).all()
    out2, st2 = lcla.forward(q, k, v, c, s, spec.block_len, spec.eps, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(out, out2) and torch.equal(st, st2)
    print(f"{name}: worst sampled output excess {worst:.2e} (bar 2e-3); state S {s_err:.2e}, z {z_err:.2e} "
          f"(bar 1e-5), relative Frobenius {fro:.2e}")


def test_empty_sequence_zeroes_state():
    q = torch.empty((1, 0, 2, 32), dtype=torch.bfloat16, device="cuda")
    c = torch.empty((0, 16), dtype=torch.float32, device="cuda")
    st = torch.full((1, 2, 33, 32), 7.0, device="cuda")
    out, st = lcla.forward(q, q, q, c, c, 4, state_out=st)
    torch.cuda.synchronize()
    assert out.numel() == 0 and torch.all(st == 0)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_guard_regions_untouched(dtype):
    """Outputs and state written exactly in bounds: canaries around them stay."""
    spec = Spec("guard", 2, 3, 1234, 32, 100, dtype, 77)
    inp = make_inputs(spec, threads=1)
    q, k, v, c, s = inputs_to_dev(inp)
    tdt = q.dtype
    pad = 4096
    n = q.numel()
    big = torch.full((n + 2 * pad,), 123.0, dtype=tdt, device="cuda")
    out = big[pad:pad + n].view(q.shape)
    sbig = torch.full((2 * 3 * 33 * 32 + 2 * pad,), -5.0, device="cuda")
    st = sbig[pad:pad + 2 * 3 * 33 * 32].view(2, 3, 33, 32)
    lcla.forward(q, k, v, c, s, spec.block_len, out=out, state_out=st)
    torch.cuda.synchronize()
    assert torch.all(big[:pad] == 123.0) and torch.all(big[pad + n:] == 123.0)
    assert torch.all(sbig[:pad] == -5.0) and torch.all(sbig[-pad:] == -5.0)
    ref, ref_st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, 100, spec.eps)
    check_outputs(host(out), ref, dtype, "guarded")
    check_state(host(st), ref_st, "guarded state")


def test_side_stream_and_determinism():
    spec = Spec("det", 1, 6, 20000, 32, 3000, "bf16", 5)
    inp = make_inputs(spec, threads=2)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        a, sa = run_gpu(inp, stream=side)
    b, sb = run_gpu(inp)
    assert torch.equal(a, b) and torch.equal(sa, sb)


def test_batch_entries_are_independent():
    """Changing batch entry 1 leaves batch entry 0 bit-identical (state isolation)."""
    spec = Spec("iso", 2, 4, 3000, 32, 700, "bf16", 11)
    inp = make_inputs(spec, threads=1)
    a, sa = run_gpu(inp)
    inp.q[1] = inp.q[1][::-1]
    inp.v[1] = inp.v[1][::-1]
    b, sb = run_gpu(inp)
    assert torch.equal(a[0], b[0]) and torch.equal(sa[0], sb[0])
    assert not torch.equal(a[1], b[1])


@pytest.mark.parametrize("name", ["fwd480p_bf16", "robust_bf16_L4680"])
def test_repeated_calls_bit_identical(name):
    """Eight back-to-back calls on the same inputs give bit-identical outputs
    and states.  The kernels reduce in a fixed order, so any difference is a
    race between pipeline roles (a buffer reused before its reader is done)."""
    spec = NAMED[name]
    inp = make_inputs(spec)
    q, k, v, c, s = inputs_to_dev(inp)
    ws = torch.empty(lcla.forward_workspace_bytes(spec.B, spec.H, spec.N, 32, spec.block_len, 0),
                     dtype=torch.uint8, device="cuda")
    out0, st0 = lcla.forward(q, k, v, c, s, spec.block_len, spec.eps, workspace=ws)
    out0, st0 = out0.clone(), st0.clone()
    for _ in range(7):
        out, st = lcla.forward(q, k, v, c, s, spec.block_len, spec.eps, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(st, st0), "state differs between identical calls"
        assert torch.equal(out, out0), "output differs between identical calls"


def _random_offsets(N, nblocks, seed, min_len=1):
    rng = np.random.default_rng(seed)
    cuts = np.sort(rng.choice(np.arange(min_len, N - min_len + 1), size=nblocks - 1, replace=False))
    return [0] + [int(c) for c in cuts] + [N]


FRAME = 130   # tokens per latent frame in the small explicit-block cases
BLOCK_CASES = [  # (B, H, N, offsets, dtype, dist)
    # first block one latent frame longer than the others (4 + 3 + 3 + 3 frames)
    (1, 6, 13 * FRAME, [0, 4 * FRAME, 7 * FRAME, 10 * FRAME, 13 * FRAME], "bf16", "normal"),
    (2, 3, 13 * FRAME, [0, 4 * FRAME, 7 * FRAME, 10 * FRAME, 13 * FRAME], "f32", "laplace_negrows"),
    # random lengths: single tokens, blocks shorter than a tile, long blocks
    (1, 5, 3000, _random_offsets(3000, 23, 7), "bf16", "laplace_negrows"),
    (1, 4, 2000, _random_offsets(2000, 31, 8), "f32", "normal"),
    (2, 7, 1500, [0, 1, 2, 3, 64, 65, 200, 1000, 1499, 1500], "bf16", "normal"),
    # one block; one block per token; more than 256 blocks (chunked scan)
    (1, 2, 300, [0, 300], "bf16", "normal"),
    (1, 2, 150, list(range(151)), "f32", "normal"),
    (1, 3, 5000, _random_offsets(5000, 300, 9), "bf16", "laplace_negrows"),
]


@pytest.mark.parametrize("B,H,N,offs,dtype,dist", BLOCK_CASES,
                         ids=[f"case{i}" for i in range(len(BLOCK_CASES))])
def test_explicit_blocks_full(B, H, N, offs, dtype, dist):
    """lcla_forward_blocks against the oracle's blocks route (the step route
    chained over the given blocks), every output and the state."""
    spec = Spec("blocks", B, H, N, 32, N, dtype, 500 + len(offs), qk_dist=dist, v_sigma=2.0)
    inp = make_inputs(spec, threads=1)
    q, k, v, c, s = inputs_to_dev(inp)
    o = torch.tensor(offs, dtype=torch.int32, device="cuda")
    out, st = lcla.forward_blocks(q, k, v, c, s, o, spec.eps)
    torch.cuda.synchronize()
    ref, ref_st = oracle.blocks(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, offs, spec.eps)
    check_outputs(host(out), ref, dtype, f"blocks {offs[:6]}...")
    check_state(host(st), ref_st, f"blocks state {offs[:6]}...")


def test_explicit_blocks_uniform_match_forward():
    """Uniform offsets give the uniform forward's results (both rounded to
    bf16, one ulp apart at most)."""
    spec = Spec("blocks_uniform", 1, 9, 4000, 32, 700, "bf16", 61, qk_dist="laplace_negrows", v_sigma=2.0)
    inp = make_inputs(spec, threads=1)
    q, k, v, c, s = inputs_to_dev(inp)
    offs = list(range(0, spec.N, spec.block_len)) + [spec.N]
    a, sa = lcla.forward(q, k, v, c, s, spec.block_len, spec.eps)
    b, sb = lcla.forward_blocks(q, k, v, c, s, torch.tensor(offs, dtype=torch.int32, device="cuda"), spec.eps)
    torch.cuda.synchronize()
    check_outputs(host(b), host(a), "bf16", "blocks vs uniform forward", ulps=1.0)
    check_state(host(sb), host(sa), "blocks vs uniform state")


def test_explicit_blocks_480p_first_block_longer():
    """The 480p-like forward (21 latent frames of 30 x 52 tokens) cut as a
    first block of 4 frames, then 3-frame blocks and a 2-frame tail, at full
    size in the launch configuration the benchmark uses, every output against
    the oracle."""
    spec = NAMED["fwd480p_bf16"]
    F = 30 * 52
    offs = [0, 4 * F] + [4 * F + 3 * F * i for i in range(1, 6)] + [spec.N]
    assert offs[-2] < spec.N and len(offs) == 8
    inp = make_inputs(spec)
    q, k, v, c, s = inputs_to_dev(inp)
    out, st = lcla.forward_blocks(q, k, v, c, s, torch.tensor(offs, dtype=torch.int32, device="cuda"), spec.eps)
    torch.cuda.synchronize()
    ref, ref_st = oracle.blocks(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, offs, spec.eps)
    check_outputs(host(out), ref, "bf16", "480p explicit blocks")
    check_state(host(st), ref_st, "480p explicit blocks state")
