"""A numpy model of the arithmetic of the bf16 tensor-core pass C, checked
against the fp64 oracle on small seeded cases (no GPU).

Pass C computes out[c] = (P q~)[c] / (z . phi(q) + eps) with (lcla_tc.cuh):
* q~ = the rotated ReLU query, rotated in fp32 and rounded once to fp16;
* P~ = each prefix row P[c] times the power of two that brings the row's
  largest magnitude below 2^14, as fp16 hi + lo at head dim 32 and as one fp16
  term at head dim 64 (two key halves);
* the product accumulated in fp32, then times the row's inverse scale and
  1 / (z . phi(q) + eps) in fp32, rounded to bf16.
The prefixes are the fp32 sums the scan produces (the oracle's fp64 prefixes
rounded to fp32 stand in for them).  The model checks that this arithmetic
keeps the worst output excess (beyond the output's own half-ulp, against the
largest output of its row: the GPU tests' metric) below half the 2e-3 bar on
robustness-style inputs -- Laplace q and k with negative rows, v of scale 2 --
and that the one-term prefix at head dim 64 stays within the same margin.
A second model restates pass A's key operand (bf16 hi + lo of the rotated key,
fp32 accumulation per 64-token tile) and checks the carried state against
its 1e-5 bar, with and without the lo term.
It models the operand roundings, not the tensor core's accumulation order."""
import numpy as np
import pytest

import oracle
from workloads import Spec, bf16_bits_to_f32, f64_to_bf16_bits, make_inputs


def bf16(x):
    return bf16_bits_to_f32(f64_to_bf16_bits(np.asarray(x, np.float64))).astype(np.float64)


def f16(x):
    return np.asarray(x, np.float64).astype(np.float16).astype(np.float64)


def f32(x):
    return np.asarray(x, np.float64).astype(np.float32).astype(np.float64)


def row_scale(m):
    """2^(14 - e) for m = f 2^e, f in [0.5, 1): the row's largest entry times it is below 2^14."""
    _, e = np.frexp(np.where(m > 0, m, 1.0))
    return np.where(m > 0, np.ldexp(1.0, 14 - e), 1.0)


def model_pass_c(inp, L, eps, hilo):
    spec = inp.spec
    d = spec.d
    _, _, pre = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, L, eps,
                                  want_out=False, want_prefix=True)
    pre = f32(pre)[0]                                          # [H, nb, d+1, d]
    q = inp.as_f32("q")[0].astype(np.float64)                  # [N, H, d]
    c = inp.rope_cos.astype(np.float64)[:, None, :]
    s = inp.rope_sin.astype(np.float64)[:, None, :]
    fq = np.maximum(q, 0.0)
    a, b = fq[..., 0::2], fq[..., 1::2]
    qr = np.empty_like(fq)
    qr[..., 0::2] = f32(a * c - b * s)
    qr[..., 1::2] = f32(a * s + b * c)
    q16 = f16(qr)
    blk = np.arange(spec.N) // L
    P = np.transpose(pre[:, blk], (1, 0, 2, 3))               # [N, H, d+1, d]
    S, z = P[:, :, :d, :], P[:, :, d, :]
    sc = row_scale(np.abs(S).max(axis=3))                     # [N, H, c]
    Ps = S * sc[..., None]
    hi = f16(Ps)
    acc = np.einsum("nhce,nhe->nhc", hi, q16)
    if hilo:
        acc = acc + np.einsum("nhce,nhe->nhc", f16(Ps - hi), q16)
    acc = f32(acc)
    den = f32(np.einsum("nhe,nhe->nh", fq, z)) + eps
    g = f32(1.0 / f32(den))
    return bf16(f32(acc * (1.0 / sc)) * g[..., None])


def excess(out, ref):
    half_ulp = 0.5 * np.abs(bf16(np.maximum(np.abs(out), np.abs(ref)))) * 2.0 ** -7
    return (np.abs(out - ref) - half_ulp) / np.maximum(np.abs(ref).max(-1, keepdims=True), 1e-300)


@pytest.mark.parametrize("d,H,L,hilo", [(32, 4, 512, True), (32, 4, 64, True), (64, 2, 512, False)])
def test_pass_c_operand_precision_within_half_the_bar(d, H, L, hilo):
    spec = Spec(f"precision_model_d{d}_L{L}", 1, H, 4096, d, L, "bf16", 21 + d + L,
                qk_dist="laplace_negrows", v_sigma=2.0, rope="1d")
    inp = make_inputs(spec)
    ref = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, L, spec.eps)[0][0]
    out = model_pass_c(inp, L, spec.eps, hilo)
    assert np.isfinite(out).all()
    worst = float(excess(out, ref).max())
    assert worst < 1e-3, worst


def test_model_detects_a_coarser_query_operand():
    # the same model with the query rounded to bf16 instead of fp16 (8 significant bits instead of 11) must
    # move the worst excess up by a clear factor: the check above is sensitive to the operand's precision
    spec = Spec("precision_model_bf16q", 1, 4, 4096, 32, 512, "bf16", 77,
                qk_dist="laplace_negrows", v_sigma=2.0, rope="1d")
    inp = make_inputs(spec)
    ref = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, 512, spec.eps)[0][0]
    fine = float(excess(model_pass_c(inp, 512, spec.eps, True), ref).max())
    global f16
    saved = f16
    try:
        f16 = bf16   # every fp16 rounding of the model becomes a bf16 rounding
        coarse = float(excess(model_pass_c(inp, 512, spec.eps, True), ref).max())
    finally:
        f16 = saved
    assert coarse > 3 * fine, (fine, coarse)


def model_pass_a_state(inp, hilo):
    """Pass A's products for the whole sequence as one block: S[c][e] = sum_t v[t][c] k~[t][e] with v as
    stored (bf16, exact), k~ = the rotated ReLU key in fp32 split into bf16 hi (+ lo), products exact and
    accumulated in fp32 over tiles of 64 tokens (the tensor core's fp32 accumulator, one tile at a time)."""
    k = inp.as_f32("k")[0].astype(np.float64)                  # [N, H, d]
    v = inp.as_f32("v")[0].astype(np.float64)
    c = inp.rope_cos.astype(np.float64)[:, None, :]
    s = inp.rope_sin.astype(np.float64)[:, None, :]
    fk = np.maximum(k, 0.0)
    a, b = fk[..., 0::2], fk[..., 1::2]
    kr = np.empty_like(fk)
    kr[..., 0::2] = f32(a * c - b * s)
    kr[..., 1::2] = f32(a * s + b * c)
    hi = bf16(kr)
    parts = [hi, bf16(kr - hi)] if hilo else [hi]
    N, H, d = k.shape
    S = np.zeros((H, d, d))
    for t0 in range(0, N, 64):
        tile = sum(np.einsum("thc,the->hce", v[t0:t0 + 64], p[t0:t0 + 64]) for p in parts)
        S = f32(S + tile)
    return S


def test_pass_a_needs_the_hi_lo_key_split_for_the_state_bar():
    # the carried state must hold 1e-5 (max |dS| / max |S|): with the bf16 hi + lo key operand the model stays
    # well inside it, with the hi term alone it does not
    spec = Spec("precision_model_state", 1, 4, 8192, 32, 8192, "bf16", 91,
                qk_dist="laplace_negrows", v_sigma=2.0, rope="1d")
    inp = make_inputs(spec)
    _, st, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, spec.block_len, spec.eps,
                                 want_out=False)
    S_ref = st[0, :, :32, :]
    err = lambda S: float(np.max(np.abs(S - S_ref)) / np.max(np.abs(S_ref)))
    assert err(model_pass_a_state(inp, True)) < 5e-6
    assert err(model_pass_a_state(inp, False)) > 1e-5
