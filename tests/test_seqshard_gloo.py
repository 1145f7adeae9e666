"""Sequence sharding's host logic, on CPU with gloo ranks.

A sequence cut into runs of whole blocks, one per rank, needs from the ranks
before it only their summed state.  Here each rank computes its part with the
fp64 oracle (the library's kernels need a GPU): the total over its tokens,
one all-gather of the totals through the product's ``gather_totals``, then its
outputs from the state carried in.  The concatenated outputs and the final
state must equal the oracle's one-shot forward.  This pins ``shard_bounds``
(ranges start on block boundaries), the rank order of the gathered totals, and
the carry algebra that ``lcla_shard_end`` runs on the GPU."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _spec(N, L, dtype):
    from workloads import Spec
    return Spec("shard", 2, 3, N, 32, L, dtype, 31, qk_dist="laplace_negrows", v_sigma=2.0)


def _state_in(B, H, d):
    rng = np.random.default_rng(5)
    st = rng.standard_normal((B, H, d + 1, d))
    st[:, :, -1, :] = np.abs(st[:, :, -1, :]) * 20
    return st


def _worker(rank, world, port, out_dir, N, L, dtype):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import oracle
    from block_causal_relu_b200.seqshard import gather_totals, shard_bounds
    from workloads import make_inputs
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        spec = _spec(N, L, dtype)
        inp = make_inputs(spec, threads=1)
        t0, t1 = shard_bounds(N, L, world)[rank]
        sl = slice(t0, t1)
        args = (inp.q[:, sl], inp.k[:, sl], inp.v[:, sl], inp.rope_cos[sl], inp.rope_sin[sl])
        B, H, d = spec.B, spec.H, spec.d
        if t1 > t0:
            _, total, _ = oracle.recurrence(*args, L, spec.eps, want_out=False)
        else:
            total = np.zeros((B, H, d + 1, d))
        totals = gather_totals(torch.from_numpy(total)).numpy()
        assert totals.shape == (world, B, H, d + 1, d)
        assert np.array_equal(totals[rank], total)
        carry = _state_in(B, H, d) + totals[:rank].sum(axis=0)
        final = _state_in(B, H, d) + totals.sum(axis=0)
        if t1 > t0:
            out, st, _ = oracle.recurrence(*args, L, spec.eps, state_in=carry)
            np.testing.assert_allclose(st, carry + total, rtol=1e-12, atol=1e-9)
        else:
            out = np.zeros((B, 0, H, d))
        np.save(os.path.join(out_dir, f"out{rank}.npy"), out)
        np.save(os.path.join(out_dir, f"final{rank}.npy"), final)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world,N,L,dtype", [
    (2, 600, 100, "f32"),      # 6 blocks, 3 per rank
    (3, 700, 90, "bf16"),      # 8 blocks dealt 3/3/2, ragged last block of 70
    (2, 300, 7, "f32"),        # short blocks (the chunk-mode cut on the GPU)
    (4, 250, 100, "bf16"),     # 3 blocks over 4 ranks: the last rank holds nothing
])
def test_sharded_oracle_equals_one_shot(tmp_path, world, N, L, dtype):
    sys.path.insert(0, ROOT)
    import oracle
    from workloads import make_inputs
    mp.start_processes(_worker, args=(world, free_port(), str(tmp_path), N, L, dtype), nprocs=world,
                       join=True, start_method="spawn")
    spec = _spec(N, L, dtype)
    inp = make_inputs(spec, threads=1)
    st_in = _state_in(spec.B, spec.H, spec.d)
    ref, ref_st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, L, spec.eps,
                                       state_in=st_in)
    out = np.concatenate([np.load(tmp_path / f"out{r}.npy") for r in range(world)], axis=1)
    assert out.shape == ref.shape
    scale = np.abs(ref).max(axis=-1, keepdims=True) + 1e-300
    assert (np.abs(out - ref) / scale).max() < 1e-11
    finals = [np.load(tmp_path / f"final{r}.npy") for r in range(world)]
    for f in finals[1:]:
        assert np.array_equal(f, finals[0])          # one summation order on every rank
    np.testing.assert_allclose(finals[0], ref_st, rtol=1e-11, atol=1e-9)


def test_shard_bounds():
    sys.path.insert(0, ROOT)
    from block_causal_relu_b200.seqshard import shard_bounds
    for N, L, R in [(32760, 4680, 2), (32760, 4680, 8), (848320, 10560, 8), (100, 30, 3), (0, 5, 2),
                    (7, 1, 7), (5, 10, 3), (65536, 64, 8)]:
        b = shard_bounds(N, L, R)
        assert len(b) == R
        assert b[0][0] == 0 and b[-1][1] == N
        for (a0, a1), (c0, _) in zip(b, b[1:]):
            assert a1 == c0 and a0 <= a1                 # contiguous, in order
        nblk = []
        for t0, t1 in b:
            assert t0 % L == 0 or t0 == N                # starts on a block boundary
            assert t1 % L == 0 or t1 == N
            nblk.append(-(-(t1 - t0) // L))
        assert max(nblk) - min(nblk) <= 1                # balanced by block count
        assert sum(nblk) == -(-N // L)
    with pytest.raises(ValueError):
        shard_bounds(10, 0, 2)
    with pytest.raises(ValueError):
        shard_bounds(10, 5, 0)


def test_gather_totals_single_process_is_one_rank():
    sys.path.insert(0, ROOT)
    from block_causal_relu_b200.seqshard import gather_totals
    t = torch.arange(12, dtype=torch.float32).reshape(1, 1, 3, 4)
    g = gather_totals(t)
    assert g.shape == (1, 1, 1, 3, 4) and torch.equal(g[0], t)
