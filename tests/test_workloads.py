"""The seeded input generators: rounding, determinism, distributions, tables,
and the named workload shapes."""
import numpy as np
import pytest
import torch

from workloads import (NAMED, Spec, bf16_bits_to_f32, f64_to_bf16_bits, make_inputs,
                       make_tables, rope_table_1d, rope_table_3d)


def test_bf16_rounding_matches_torch_on_float32_values():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    ours = f64_to_bf16_bits(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_rounding_ties_and_double_rounding():
    one = 1.0
    ulp = 2.0 ** -7
    # exact ties go to the even neighbour
    assert bf16_bits_to_f32(f64_to_bf16_bits(np.array([one + ulp / 2])))[0] == 1.0
    assert bf16_bits_to_f32(f64_to_bf16_bits(np.array([one + 3 * ulp / 2])))[0] == one + 2 * ulp
    # just above a tie rounds up even when float32 rounding would land on the tie
    x = one + ulp / 2 + 2.0 ** -40
    assert bf16_bits_to_f32(f64_to_bf16_bits(np.array([x])))[0] == one + ulp
    assert bf16_bits_to_f32(f64_to_bf16_bits(np.array([-x])))[0] == -(one + ulp)


def test_generation_is_deterministic_and_thread_independent():
    spec = Spec("t", 1, 3, 3000, 32, 100, "bf16", 9, qk_dist="laplace_negrows")
    a = make_inputs(spec, threads=1)
    b = make_inputs(spec, threads=4)
    for n in ("q", "k", "v"):
        assert np.array_equal(getattr(a, n), getattr(b, n))
    c = make_inputs(Spec("t", 1, 3, 3000, 32, 100, "bf16", 10, qk_dist="laplace_negrows"))
    assert not np.array_equal(a.q, c.q)
    assert not np.array_equal(a.q, a.k)


def test_distributions():
    spec = Spec("t", 1, 16, 4096, 32, 64, "f32", 4, qk_dist="laplace_negrows", v_sigma=2.0)
    inp = make_inputs(spec)
    rows = inp.q.reshape(-1, 32)
    neg = (rows <= 0).all(axis=1)
    assert abs(neg.mean() - (0.3 + 0.7 * 2.0 ** -32)) < 0.01
    assert abs(np.abs(inp.k).mean() - 1.0) < 0.02           # Laplace(0, 1): E|x| = 1
    assert abs(inp.v.std() - 2.0) < 0.02
    n = make_inputs(Spec("t", 1, 8, 4096, 32, 64, "bf16", 5))
    qf = n.as_f32("q")
    assert abs(qf.std() - 1.0) < 0.01 and abs(qf.mean()) < 0.01


def test_tables():
    c, s = rope_table_1d(100, 32)
    assert c.shape == (100, 16) and c.dtype == np.float32
    assert np.allclose(c[0], 1) and np.allclose(s[0], 0)
    assert np.allclose(c.astype(np.float64) ** 2 + s.astype(np.float64) ** 2, 1, atol=1e-6)
    assert np.isclose(np.arctan2(s[1, 1], c[1, 1]), 10000.0 ** (-2 / 32))
    c3, s3 = rope_table_3d(3, 4, 5)
    assert c3.shape == (60, 16)
    n = 2 * 20 + 3 * 5 + 4                       # frame 2, row 3, col 4
    def ang_is(p, a):
        return np.isclose(c3[n, p], np.cos(a), atol=1e-6) and np.isclose(s3[n, p], np.sin(a), atol=1e-6)
    assert ang_is(0, 2.0)                        # t pairs 0..3
    assert ang_is(4, 3.0)                        # h pairs 4..9
    assert ang_is(10, 4.0)                       # w pairs 10..15
    assert ang_is(5, 3.0 * 10000.0 ** (-2 / 12))
    assert ang_is(1, 2.0 * 10000.0 ** (-2 / 8))
    # a slice of a spec's tables equals the tables at absolute positions
    spec = NAMED["stream_bf16"]
    full = make_tables(spec)
    part = make_tables(spec, 4680 * 3, 4680)
    assert np.array_equal(full[0][4680 * 3:4680 * 4], part[0])
    assert np.array_equal(full[1][4680 * 3:4680 * 4], part[1])


def test_named_workloads():
    assert NAMED["tiny_f32"].nblocks == 4
    s = NAMED["fwd480p_bf16"]
    assert (s.N, s.block_len, s.nblocks, s.H) == (32760, 4680, 7, 70)
    s = NAMED["stream_bf16"]
    assert (s.B, s.N, s.nblocks, s.N - 13 * 4680) == (2, 63960, 14, 3120)
    s = NAMED["minute_bf16"]
    assert (s.N, s.block_len, s.nblocks, s.N - 80 * 10560) == (848320, 10560, 81, 3520)
    for L in (1, 64, 1560, 4680, 65536):
        for dt in ("f32", "bf16"):
            s = NAMED[f"robust_{dt}_L{L}"]
            assert (s.B, s.H, s.N, s.qk_dist, s.v_sigma) == (1, 16, 65536, "laplace_negrows", 2.0)
