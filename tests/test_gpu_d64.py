"""Head dim 64 on the GPU against the fp64 oracle.

d = 64 runs in block mode for every block length: bf16 on the tensor-core
passes (each 64-dim head as two 32-dim virtual heads), fp32 on the generic
CUDA-core passes.  Small cases span several 32-token tiles, ragged tails, blocks shorter
than a tile and more than 256 blocks (the chunked scan); the 480p-like latent
at head dim 64 (35 heads x 64 = the same 2240 width) runs at full size and is
compared on sampled rows plus the full state.  The other entry points
(explicit blocks, streaming steps, sequence sharding) are checked at d = 64
too."""
import numpy as np
import pytest
import torch

import block_causal_relu_b200 as lcla
import oracle
from gpu_util import dev, host, inputs_to_dev, sample_rows
from parity import check_outputs, check_state
from workloads import NAMED, Spec, make_inputs

pytestmark = pytest.mark.gpu

D = 64

SMALL = [  # (B, H, N, block_len, dtype, dist)
    (1, 2, 1000, 256, "bf16", "normal"),
    (2, 3, 777, 100, "f32", "laplace_negrows"),
    (1, 2, 300, 1, "f32", "normal"),              # 300 one-token blocks: chunked scan
    (1, 3, 129, 7, "bf16", "laplace_negrows"),
    (1, 4, 5000, 5000, "bf16", "normal"),          # one block
    (2, 1, 65, 64, "f32", "normal"),
    (1, 5, 2000, 33, "bf16", "normal"),
    (1, 2, 1, 1, "f32", "normal"),
    (1, 1, 300, 100, "bf16", "normal"),            # one head: its quad's last two virtual heads are past H
    (3, 2, 129, 64, "bf16", "laplace_negrows"),    # batch 3, ragged last tile
    (1, 3, 70, 5, "bf16", "normal"),               # 14 blocks shorter than a tile
]


@pytest.mark.parametrize("B,H,N,L,dtype,dist", SMALL)
def test_small_cases_full(B, H, N, L, dtype, dist):
    spec = Spec("d64", B, H, N, D, L, dtype, 2000 + N + L, qk_dist=dist, v_sigma=2.0)
    inp = make_inputs(spec, threads=2)
    q, k, v, c, s = inputs_to_dev(inp)
    assert not lcla.plan_info(B, H, N, D, L, lcla.BF16 if dtype == "bf16" else lcla.F32)["chunk_mode"]
    out, st = lcla.forward(q, k, v, c, s, L, spec.eps)
    torch.cuda.synchronize()
    assert tuple(st.shape) == (B, H, D + 1, D)
    ref, ref_st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, L, spec.eps)
    check_outputs(host(out), ref, dtype, f"d64 {spec}")
    check_state(host(st), ref_st, f"d64 state {spec}")
    if N * N * H * B <= 2e7:
        msk = oracle.masked(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, L, spec.eps)
        check_outputs(host(out), msk, dtype, f"d64 vs masked {spec}")


def test_480p_d64_sampled():
    spec = NAMED["fwd480p_d64_bf16"]
    inp = make_inputs(spec)
    q, k, v, c, s = inputs_to_dev(inp)
    out, st = lcla.forward(q, k, v, c, s, spec.block_len, spec.eps)
    torch.cuda.synchronize()
    rows = sample_rows(spec.N, spec.block_len, 2048, seed=7)
    ref, ref_st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, spec.block_len,
                                       spec.eps, rows=rows)
    check_outputs(host(out[:, torch.from_numpy(rows).cuda()]), ref, "bf16", "480p d64 vs oracle")
    check_state(host(st), ref_st, "480p d64 state")


def test_explicit_blocks_d64():
    spec = Spec("d64blk", 1, 3, 2500, D, 500, "bf16", 2101)
    inp = make_inputs(spec, threads=2)
    q, k, v, c, s = inputs_to_dev(inp)
    offs = np.array([0, 700, 1200, 1201, 2500], np.int32)    # a first block longer, a one-token block
    out, st = lcla.forward_blocks(q, k, v, c, s, torch.from_numpy(offs).cuda(), spec.eps)
    torch.cuda.synchronize()
    ref, ref_st = oracle.blocks(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, offs, spec.eps)
    check_outputs(host(out), ref, "bf16", "d64 explicit blocks")
    check_state(host(st), ref_st, "d64 explicit blocks state")


@pytest.mark.parametrize("dtype,L", [("bf16", 700), ("f32", 16)])
def test_step_chain_d64(dtype, L):
    spec = Spec("d64step", 2, 2, 4 * L, D, L, dtype, 2200 + L, qk_dist="laplace_negrows", v_sigma=2.0)
    inp = make_inputs(spec, threads=2)
    q, k, v, c, s = inputs_to_dev(inp)
    state = torch.zeros((2, 2, D + 1, D), device="cuda")
    outs = []
    for t0 in range(0, spec.N, L):
        sl = slice(t0, t0 + L)
        blk = [x[:, sl].contiguous() for x in (q, k, v)] + [c[sl].contiguous(), s[sl].contiguous()]
        before = state.clone()
        o_peek = lcla.step(*blk, state, save=False)
        torch.cuda.synchronize()
        assert torch.equal(state, before), "save=0 wrote the state"
        outs.append(lcla.step(*blk, state, save=True))
        torch.cuda.synchronize()
        assert torch.equal(o_peek, outs[-1])
    ref, ref_st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, L, spec.eps)
    check_outputs(host(torch.cat(outs, dim=1)), ref, dtype, f"d64 step chain {dtype} L{L}")
    check_state(host(state), ref_st, "d64 step chain state")


def test_sharded_d64():
    from block_causal_relu_b200.seqshard import shard_bounds
    spec = Spec("d64shard", 1, 3, 3000, D, 400, "bf16", 2301)
    inp = make_inputs(spec, threads=2)
    q, k, v, c, s = inputs_to_dev(inp)
    rng = np.random.default_rng(3)
    st0 = rng.standard_normal((1, 3, D + 1, D)).astype(np.float32)
    st0[:, :, -1, :] = np.abs(st0[:, :, -1, :]) * 30
    parts, totals, wss = [], [], []
    for t0, t1 in shard_bounds(spec.N, spec.block_len, 3):
        sl = slice(t0, t1)
        part = [x[:, sl].contiguous() for x in (q, k, v)] + [c[sl].contiguous(), s[sl].contiguous()]
        total, ws = lcla.shard_begin(part[1], part[2], part[3], part[4], spec.block_len)
        parts.append(part)
        totals.append(total)
        wss.append(ws)
    g = torch.stack(totals)
    res = [lcla.shard_end(*pt, spec.block_len, g, r, wss[r], spec.eps, state_in=dev(st0))
           for r, pt in enumerate(parts)]
    torch.cuda.synchronize()
    ref, ref_st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, spec.block_len,
                                       spec.eps, state_in=st0.astype(np.float64))
    check_outputs(host(torch.cat([o for o, _ in res], dim=1)), ref, "bf16", "d64 sharded")
    check_state(host(res[0][1]), ref_st, "d64 sharded state")
    assert all(torch.equal(st, res[0][1]) for _, st in res)


def test_d64_repeated_calls_bit_identical():
    spec = Spec("d64det", 2, 5, 3000, D, 700, "bf16", 2401, qk_dist="laplace_negrows", v_sigma=2.0)
    inp = make_inputs(spec, threads=2)
    q, k, v, c, s = inputs_to_dev(inp)
    ref_out, ref_st = lcla.forward(q, k, v, c, s, spec.block_len, spec.eps)
    for _ in range(5):
        out, st = lcla.forward(q, k, v, c, s, spec.block_len, spec.eps)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out) and torch.equal(st, ref_st)
