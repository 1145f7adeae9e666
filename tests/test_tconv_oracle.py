"""The temporal-convolution oracle against a plain loop of its definition and
the facts that follow from it (no GPU)."""
import numpy as np
import pytest

from oracle.tconv import temporal_conv
from workloads import f64_to_bf16_bits, bf16_bits_to_f32


def loop_definition(x, S, w, b, cache):
    """y[b, f, s, c] = w[0, c] x[b, f, s, c] + w[1, c] x[b, f-1, s, c] + bias[c],
    frame -1 = cache (zeros without one), element by element."""
    B, N, C = x.shape
    F = N // S
    y = np.zeros((B, N, C))
    for bb in range(B):
        for f in range(F):
            for s in range(S):
                for c in range(C):
                    prev = (x[bb, (f - 1) * S + s, c] if f > 0 else
                            (0.0 if cache is None else cache[bb, s, c]))
                    y[bb, f * S + s, c] = (w[0, c] * x[bb, f * S + s, c] + w[1, c] * prev
                                           + (0.0 if b is None else b[c]))
    return y


def _case(seed, B=2, F=3, S=5, C=8, with_cache=True, with_bias=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, F * S, C)).astype(np.float32)
    w = rng.standard_normal((2, C)).astype(np.float32)
    b = rng.standard_normal(C).astype(np.float32) if with_bias else None
    cache = rng.standard_normal((B, S, C)).astype(np.float32) if with_cache else None
    return x, w, b, cache


@pytest.mark.parametrize("with_cache,with_bias", [(True, True), (False, True), (True, False), (False, False)])
def test_against_loop(with_cache, with_bias):
    x, w, b, cache = _case(1, with_cache=with_cache, with_bias=with_bias)
    y, last = temporal_conv(x, 5, w, b, cache)
    ref = loop_definition(x.astype(np.float64), 5, w.astype(np.float64),
                          None if b is None else b.astype(np.float64),
                          None if cache is None else cache.astype(np.float64))
    assert np.abs(y - ref).max() <= 1e-12 * np.abs(ref).max()
    assert np.array_equal(last, x[:, -5:].astype(np.float64))


def test_identity_and_shift():
    x, _, _, cache = _case(2)
    C = x.shape[-1]
    ident = np.stack([np.ones(C), np.zeros(C)]).astype(np.float32)
    shift = np.stack([np.zeros(C), np.ones(C)]).astype(np.float32)
    y, _ = temporal_conv(x, 5, ident, None, cache)
    assert np.array_equal(y, x.astype(np.float64))
    y, _ = temporal_conv(x, 5, shift, None, cache)
    assert np.array_equal(y[:, 5:], x[:, :-5].astype(np.float64))      # x[f - 1]
    assert np.array_equal(y[:, :5], cache.astype(np.float64))          # frame -1 is the cache


def test_streaming_equals_one_call():
    x, w, b, _ = _case(3, F=7)
    whole, last = temporal_conv(x, 5, w, b, None)
    y1, c1 = temporal_conv(x[:, :15], 5, w, b, None)
    y2, c2 = temporal_conv(x[:, 15:], 5, w, b, c1.astype(np.float32))
    assert np.abs(np.concatenate([y1, y2], axis=1) - whole).max() <= 1e-12 * np.abs(whole).max()
    assert np.array_equal(c2, last)


def test_bf16_widening_exact():
    rng = np.random.default_rng(4)
    bits = f64_to_bf16_bits(rng.standard_normal(2 * 10 * 8)).reshape(2, 10, 8)
    w = rng.standard_normal((2, 8)).astype(np.float32)
    a, _ = temporal_conv(bits, 5, w)
    b, _ = temporal_conv(bf16_bits_to_f32(bits), 5, w)
    assert np.array_equal(a, b)
