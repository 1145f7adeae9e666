"""Sequence-sharded forward on one GPU: the ranks run one after another.

Each rank's ``shard_begin`` (pass A and the rank's state total) runs first,
the totals are stacked in rank order as the all-gather would leave them, then
each rank's ``shard_end`` (carry-in kernel, scan, pass C).  No kernel waits on
another rank, so running the ranks in sequence on one device exercises every
kernel of the multi-GPU path.  The concatenated outputs must match the fp64
oracle's one-shot forward within the parity bar, every rank must write the
same final state bit for bit, and that state must match the oracle's."""
import numpy as np
import pytest
import torch

import block_causal_relu_b200 as lcla
import oracle
from block_causal_relu_b200.seqshard import forward_sharded, shard_bounds
from gpu_util import dev, host, inputs_to_dev, sample_rows
from parity import check_outputs, check_state
from workloads import NAMED, Spec, make_inputs

pytestmark = pytest.mark.gpu


def run_ranks(q, k, v, c, s, L, world, eps, state_in=None):
    """Every rank's two calls, in sequence; returns (outputs per rank, final states per rank)."""
    N = q.shape[1]
    bounds = shard_bounds(N, L, world)
    parts, totals, wss = [], [], []
    for t0, t1 in bounds:
        sl = slice(t0, t1)
        part = [x[:, sl].contiguous() for x in (q, k, v)] + [c[sl].contiguous(), s[sl].contiguous()]
        total, ws = lcla.shard_begin(part[1], part[2], part[3], part[4], L)
        parts.append(part)
        totals.append(total)
        wss.append(ws)
    gathered = torch.stack(totals)
    outs, finals = [], []
    for r, part in enumerate(parts):
        o, st = lcla.shard_end(*part, L, gathered, r, wss[r], eps, state_in=state_in)
        outs.append(o)
        finals.append(st)
    torch.cuda.synchronize()
    return outs, finals


def state_in_for(B, H, seed=7):
    rng = np.random.default_rng(seed)
    st = rng.standard_normal((B, H, 33, 32)).astype(np.float32)
    st[:, :, -1, :] = np.abs(st[:, :, -1, :]) * 30
    return st


CASES = [
    # (B, H, N, L, dtype, world)
    (1, 8, 8192, 1024, "bf16", 2),       # tensor cores, whole blocks per rank
    (2, 5, 5000, 700, "f32", 3),         # CUDA cores, ragged last block
    (1, 6, 3000, 256, "bf16", 5),        # several blocks per rank, ragged
    (2, 4, 2048, 16, "bf16", 4),         # chunk mode (block_len < 64)
    (1, 3, 1000, 7, "f32", 3),           # chunk mode, blocks straddling tiles
    (1, 8, 2500, 1000, "bf16", 4),       # 3 blocks over 4 ranks: one rank empty
]


@pytest.mark.parametrize("B,H,N,L,dtype,world", CASES)
def test_sharded_equals_oracle(B, H, N, L, dtype, world):
    spec = Spec("shard", B, H, N, 32, L, dtype, 41, qk_dist="laplace_negrows", v_sigma=2.0)
    inp = make_inputs(spec, threads=4)
    q, k, v, c, s = inputs_to_dev(inp)
    st0 = state_in_for(B, H)
    outs, finals = run_ranks(q, k, v, c, s, L, world, spec.eps, state_in=dev(st0))
    out = torch.cat(outs, dim=1)
    ref, ref_st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, L, spec.eps,
                                       state_in=st0.astype(np.float64))
    check_outputs(host(out), ref, dtype, f"sharded x{world} {B}x{N}x{H} L{L} {dtype}")
    for f in finals[1:]:
        assert torch.equal(f, finals[0]), "ranks disagree on the final state"
    check_state(host(finals[0]), ref_st, "sharded final state")


def test_one_rank_equals_forward_bitwise():
    """With one rank the carry is state_in and the path is the forward's."""
    spec = Spec("shard1", 1, 8, 4096, 32, 1024, "bf16", 43)
    inp = make_inputs(spec, threads=4)
    q, k, v, c, s = inputs_to_dev(inp)
    outs, finals = run_ranks(q, k, v, c, s, 1024, 1, spec.eps)
    full, st = lcla.forward(q, k, v, c, s, 1024, spec.eps)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], full)
    assert torch.equal(finals[0], st)


@pytest.mark.parametrize("world", [2, 7])
def test_480p_sharded(world):
    """The 480p-like forward (7 blocks of 4680) over 2 and 7 ranks, against the
    one-shot GPU forward and the oracle on sampled rows."""
    spec = NAMED["fwd480p_bf16"]
    inp = make_inputs(spec)
    q, k, v, c, s = inputs_to_dev(inp)
    outs, finals = run_ranks(q, k, v, c, s, spec.block_len, world, spec.eps)
    out = torch.cat(outs, dim=1)
    full, st_full = lcla.forward(q, k, v, c, s, spec.block_len, spec.eps)
    torch.cuda.synchronize()
    check_outputs(host(out), host(full), "bf16", "sharded vs forward", ulps=1.0)
    check_state(host(finals[0]), host(st_full), "sharded state vs forward")
    rows = sample_rows(spec.N, spec.block_len, 2048, seed=5)
    ref, ref_st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, spec.block_len,
                                       spec.eps, rows=rows)
    check_outputs(host(out[:, torch.from_numpy(rows).cuda()]), ref, "bf16", "sharded vs oracle")
    check_state(host(finals[0]), ref_st, "sharded state vs oracle")


def test_forward_sharded_single_process():
    """The host driver without a process group is one rank."""
    spec = Spec("shardfs", 1, 4, 2048, 32, 512, "bf16", 44)
    inp = make_inputs(spec, threads=4)
    q, k, v, c, s = inputs_to_dev(inp)
    out, st = forward_sharded(q, k, v, c, s, 512, spec.eps)
    full, st_full = lcla.forward(q, k, v, c, s, 512, spec.eps)
    torch.cuda.synchronize()
    assert torch.equal(out, full) and torch.equal(st, st_full)


def test_state_out_may_alias_state_in():
    spec = Spec("shardalias", 1, 4, 1024, 32, 256, "f32", 45)
    inp = make_inputs(spec, threads=4)
    q, k, v, c, s = inputs_to_dev(inp)
    st0 = dev(state_in_for(1, 4, seed=9))
    total, ws = lcla.shard_begin(k, v, c, s, 256)
    gathered = total.unsqueeze(0)
    o1, st1 = lcla.shard_end(q, k, v, c, s, 256, gathered, 0, ws, spec.eps, state_in=st0)
    inplace = st0.clone()
    o2, _ = lcla.shard_end(q, k, v, c, s, 256, gathered, 0, ws, spec.eps, state_in=inplace, state_out=inplace)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(st1, inplace)
