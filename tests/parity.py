"""Parity metrics between the CUDA path and the fp64 oracle.

Output rows: the elementwise relative error is unusable because S q~ cancels
towards zero and a bf16 store alone is up to 2^-9 relative.  Each output
element o is compared with the unrounded oracle value r of the same
(b, n, h) row, scaled by that row's largest magnitude, after allowing half an
ulp of the output type at max(|o|, |r|):

    |o - r| - ulp_out(max(|o|, |r|)) / 2  <=  tol * max_c |r[b, n, h, c]|

tol = 2e-3 for bf16 inputs, 1e-5 for fp32 inputs (the stated tolerances).
A row whose oracle values are all zero (q row with no positive entry) must
come out exactly zero.

State: per (b, h), max |dS| / max |S| <= 1e-5, and the key sum z (a sum of
non-negative terms, no cancellation) elementwise relative <= 1e-5.
"""
from __future__ import annotations

import numpy as np

TOL = {"bf16": 2e-3, "f32": 1e-5}
STATE_TOL = 1e-5


def ulp(x: np.ndarray, dtype: str) -> np.ndarray:
    """Spacing of the output type at |x| (normal range)."""
    mant = 7 if dtype == "bf16" else 23
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.exp2(np.floor(np.log2(ax)) - mant)


def output_excess(o: np.ndarray, r: np.ndarray, dtype: str, ulps: float = 0.5) -> np.ndarray:
    """Per-row worst excess of the error over its allowance, divided by the
    row scale; values <= tol pass.  Rows with zero scale give 0 when exact and
    +inf otherwise.  ``ulps`` is the rounding allowance in output ulps: 1/2
    against the unrounded oracle, 1 when both sides are rounded outputs."""
    o = np.asarray(o, np.float64)
    r = np.asarray(r, np.float64)
    assert o.shape == r.shape, (o.shape, r.shape)
    scale = np.abs(r).max(axis=-1)
    err = np.abs(o - r) - ulps * ulp(np.maximum(np.abs(o), np.abs(r)), dtype)
    worst = np.maximum(err.max(axis=-1), 0.0)
    with np.errstate(divide="ignore", invalid="ignore"):
        rel = np.where(scale > 0, worst / np.where(scale > 0, scale, 1.0),
                       np.where(np.abs(o).max(axis=-1) == 0, 0.0, np.inf))
    return rel


def check_outputs(o, r, dtype: str, what: str = "", ulps: float = 0.5) -> float:
    rel = output_excess(o, r, dtype, ulps)
    worst = float(rel.max()) if rel.size else 0.0
    if not np.isfinite(o).all():
        raise AssertionError(f"{what}: non-finite outputs")
    if worst > TOL[dtype]:
        idx = np.unravel_index(int(np.argmax(rel)), rel.shape)
        raise AssertionError(f"{what}: output error {worst:.3e} > {TOL[dtype]:.0e} at row {idx}")
    return worst


def check_state(st, ref, what: str = "") -> tuple:
    st = np.asarray(st, np.float64)
    ref = np.asarray(ref, np.float64)
    assert st.shape == ref.shape, (st.shape, ref.shape)
    S, Sr = st[..., :-1, :], ref[..., :-1, :]
    z, zr = st[..., -1, :], ref[..., -1, :]
    sden = np.abs(Sr).max(axis=(-2, -1))
    s_rel = np.abs(S - Sr).max(axis=(-2, -1)) / np.where(sden > 0, sden, 1.0)
    with np.errstate(divide="ignore", invalid="ignore"):
        z_rel = np.where(zr > 0, np.abs(z - zr) / np.where(zr > 0, zr, 1.0), np.abs(z - zr))
    ws, wz = float(s_rel.max()), float(z_rel.max())
    # also the per-(b, h) relative Frobenius error of S (reported, not a bar)
    fden = np.sqrt((Sr ** 2).sum(axis=(-2, -1)))
    fro = float((np.sqrt(((S - Sr) ** 2).sum(axis=(-2, -1))) / np.where(fden > 0, fden, 1.0)).max())
    if ws > STATE_TOL or wz > STATE_TOL:
        raise AssertionError(f"{what}: state error S {ws:.3e}, z {wz:.3e} > {STATE_TOL:.0e} "
                             f"(relative Frobenius {fro:.3e})")
    return ws, wz, fro
