"""The work plan on the host: the segment map the kernels evaluate, checked for
any shape.  Segments must partition [0, N) in order; in block mode each lies in
one block of block_len tokens and every block is covered; in chunk mode tiles
hold whole blocks, so every segment starts on a block boundary.  No GPU."""
import pytest
from hypothesis import given, settings, strategies as st

import block_causal_relu_b200 as lcla


def check_plan(B, H, N, d, L, dtype):
    info = lcla.plan_info(B, H, N, d, L, dtype)
    segs = lcla.plan_segments(B, H, N, d, L, dtype)
    assert len(segs) == info["segments"]
    pos = 0
    for t0, t1, blk in segs:
        assert t0 == pos and t0 <= t1 <= N             # in order, no gap, no overlap
        pos = t1
    assert pos == N                                     # every token once
    if info["chunk_mode"]:
        T = info["tile_tokens"]
        assert d == 32 and L < 64 and T % L == 0 and T <= 64
        assert info["prefixes"] == info["segments"]
        for t0, t1, blk in segs:
            assert blk == -1
            assert t0 % T == 0 or t0 == N               # segments are runs of whole tiles of whole blocks
    else:
        nb = -(-N // L)
        assert info["prefixes"] == nb
        covered = [0] * nb
        for t0, t1, blk in segs:
            assert 0 <= blk < nb
            b0, b1 = blk * L, min(N, (blk + 1) * L)
            assert b0 <= t0 <= t1 <= b1                 # inside its block
            covered[blk] += t1 - t0
        assert covered == [min(N, (b + 1) * L) - b * L for b in range(nb)]
        # the tensor cores take bf16 in block mode (d = 32 and d = 64)
        assert info["tensor_cores"] == (dtype == lcla.BF16)


@settings(max_examples=300, deadline=None)
@given(N=st.integers(1, 200_000), L=st.integers(1, 70_000), H=st.integers(1, 80), B=st.integers(1, 4),
       d=st.sampled_from([32, 64]), dtype=st.sampled_from([lcla.BF16, lcla.F32]))
def test_segments_partition_the_sequence(N, L, H, B, d, dtype):
    if d == 64 and N // L > 20_000:   # d = 64 keeps one state per block: skip plans of huge workspaces
        return
    check_plan(B, H, N, d, L, dtype)


@pytest.mark.parametrize("B,H,N,d,L,dtype", [
    (1, 70, 32760, 32, 4680, lcla.BF16),     # 480p
    (1, 70, 848320, 32, 10560, lcla.BF16),   # minute scale, ragged last block
    (2, 70, 63960, 32, 4680, lcla.BF16),     # streaming workload as one forward
    (1, 16, 65536, 32, 1, lcla.BF16),        # token-causal reading
    (1, 16, 65536, 32, 64, lcla.F32),
    (1, 35, 32760, 64, 4680, lcla.BF16),     # head dim 64
    (1, 3, 100, 64, 7, lcla.F32),
    (3, 5, 1, 32, 1, lcla.BF16),
])
def test_named_shapes(B, H, N, d, L, dtype):
    check_plan(B, H, N, d, L, dtype)


def test_plan_segments_arguments():
    import ctypes
    a = (ctypes.c_int * 4)()
    assert lcla.lib.lcla_forward_plan_segments(1, 2, 1000, 32, 100, lcla.BF16, a, a, a, 4) == 1   # too small
    assert lcla.lib.lcla_forward_plan_segments(1, 2, 1000, 32, 100, lcla.BF16, None, a, a, 100) == 1
    assert lcla.lib.lcla_forward_plan_segments(1, 2, 1000, 48, 100, lcla.BF16, a, a, a, 100) == 2   # d = 48
