"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` handle and raises
``AssertionError`` when the oracle disagrees with the fact it checks.  They are
run on the real oracle by ``test_oracle_pins.py`` and on deliberately broken
builds of it by ``test_oracle_mutants.py`` (every broken build must fail at
least one pin).

Sources of truth used here:
* the printed non-causal formula ("Implementing Block Causal Linear Attention
  for Long Video Generation with Sana", section "The Linear Attention
  Kernel"), written out in numpy (``oracle.literal``);
* causal linear attention as a running sum over tokens (the recurrent view of
  linear attention, Katharopoulos et al. 2020, "Transformers are RNNs"), with
  the rotary embedding written as complex multiplication of interleaved pairs;
* exact rational arithmetic on dyadic inputs and quarter-turn rotary tables;
* closed forms and symmetries that follow from the definition.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

from oracle.literal import literal
from workloads import Spec, make_inputs, rope_table_1d, f64_to_bf16_bits, bf16_bits_to_f32


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------
def rows_close(a, r, tol, what=""):
    """|a - r| <= tol * max_c |r[..., c]| for every (b, n, h) row."""
    a = np.asarray(a, np.float64)
    r = np.asarray(r, np.float64)
    assert a.shape == r.shape, (what, a.shape, r.shape)
    scale = np.abs(r).max(axis=-1, keepdims=True)
    err = np.abs(a - r)
    ok = err <= tol * scale
    if not ok.all():
        idx = np.unravel_index(np.argmax(err - tol * scale), err.shape)
        raise AssertionError(f"{what}: err {err[idx]:.3e} > {tol:.1e} * {scale[idx[:-1]][0]:.3e} at {idx}")


def small(seed, B=2, H=3, N=37, d=8, L=5, dtype="f32", dist="normal"):
    spec = Spec("pin", B, H, N, d, L, dtype, seed, qk_dist=dist, v_sigma=1.0)
    return make_inputs(spec, threads=1)


def _complex_rotary(x, cos, sin):
    """Rotary embedding as complex multiplication: pair (x_2p, x_2p+1) is the
    complex number x_2p + i x_2p+1, multiplied by cos + i sin of its token."""
    z = x[..., 0::2] + 1j * x[..., 1::2]
    w = (cos.astype(np.float64) + 1j * sin.astype(np.float64))
    shape = [1] * z.ndim
    shape[1] = w.shape[0]           # tokens on axis 1 of [B, N, H, d/2]
    shape[-1] = w.shape[1]
    zr = z * w.reshape(shape)
    y = np.empty(x.shape, np.float64)
    y[..., 0::2] = zr.real
    y[..., 1::2] = zr.imag
    return y


def causal_cumsum(q, k, v, cos, sin, eps):
    """Token-causal linear attention (each token attends to itself and all
    earlier tokens) as cumulative sums of outer products, complex rotary."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    fq, fk = np.maximum(q, 0), np.maximum(k, 0)
    rq, rk = _complex_rotary(fq, cos, sin), _complex_rotary(fk, cos, sin)
    S = np.cumsum(v[..., :, None] * rk[..., None, :], axis=1)   # [B, N, H, d, d]
    z = np.cumsum(fk, axis=1)                                    # [B, N, H, d]
    num = np.einsum("bnhce,bnhe->bnhc", S, rq)
    den = np.einsum("bnhe,bnhe->bnh", z, fq)[..., None] + eps
    return num / den, S[:, -1], z[:, -1]


# ----------------------------------------------------------------------------
# pins
# ----------------------------------------------------------------------------
def pin_masked_equals_recurrence(orc):
    """The pair-by-pair definition and the block recurrence are two independent
    routes to the same numbers."""
    cases = [dict(seed=1, N=37, L=5), dict(seed=2, N=40, L=8), dict(seed=3, N=33, L=1),
             dict(seed=4, N=29, L=29), dict(seed=5, N=31, L=64),
             dict(seed=6, N=50, L=7, dtype="bf16", dist="laplace_negrows"),
             dict(seed=7, N=24, L=6, d=32), dict(seed=8, N=22, L=6, d=64),
             dict(seed=9, N=17, L=17, d=64, dtype="bf16", dist="laplace_negrows")]
    for c in cases:
        inp = small(c["seed"], N=c["N"], L=c["L"], d=c.get("d", 8), dtype=c.get("dtype", "f32"),
                    dist=c.get("dist", "normal"))
        a = orc.masked(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, c["L"], 1e-8)
        b, _, _ = orc.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, c["L"], 1e-8)
        rows_close(a, b, 1e-12, f"masked vs recurrence {c}")


def pin_single_block_equals_printed_formula(orc):
    """block_len = N is the printed non-causal formula, with the normaliser on
    the unrotated features and vk = v k_rotated^T."""
    for seed, dtype, dist, d in [(11, "f32", "normal", 8), (12, "bf16", "laplace_negrows", 8),
                                 (13, "f32", "normal", 64)]:
        inp = small(seed, N=23, d=d, dtype=dtype, dist=dist)
        ref = literal(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, 1e-8)
        rec, _, _ = orc.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, 23, 1e-8)
        rows_close(rec, ref, 1e-12, "recurrence(block_len=N) vs printed formula")
        msk = orc.masked(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, 23, 1e-8)
        rows_close(msk, ref, 1e-12, "masked(block_len=N) vs printed formula")
        # block_len beyond N is the same single block
        rec2, _, _ = orc.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, 1000, 1e-8)
        rows_close(rec2, ref, 1e-12, "recurrence(block_len>N) vs printed formula")


def pin_block_len_one_is_token_causal(orc):
    """block_len = 1 is token-causal linear attention (running sums), and the
    final state is the total sum of v k_rot^T and phi(k)."""
    for seed, d in ((21, 8), (22, 64)):
        inp = small(seed, N=41, d=d, dtype="f32")
        q, k, v = (inp.as_f32(n) for n in ("q", "k", "v"))
        ref, S, z = causal_cumsum(q, k, v, inp.rope_cos, inp.rope_sin, 1e-8)
        out, st, _ = orc.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, 1, 1e-8)
        rows_close(out, ref, 1e-12, f"block_len=1 vs running sums, d={d}")
        msk = orc.masked(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, 1, 1e-8)
        rows_close(msk, ref, 1e-12, f"masked block_len=1 vs running sums, d={d}")
        scale = np.abs(S).max()
        assert np.abs(st[:, :, :-1, :] - S).max() <= 1e-12 * scale, "state S vs running sum"
        assert np.abs(st[:, :, -1, :] - z).max() <= 1e-12 * np.abs(z).max(), "state z vs running sum"


def pin_step_chain_equals_forward(orc):
    """Feeding the blocks one at a time with save=1 reproduces the whole-
    sequence outputs and final state; save=0 leaves the state untouched."""
    inp = small(31, B=2, H=2, N=26, d=8, L=6)
    L = 6
    full, st_full, _ = orc.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, L, 1e-8)
    B, N, H, d = inp.q.shape
    state = np.zeros((B, H, d + 1, d))
    outs = []
    for t0 in range(0, N, L):
        t1 = min(N, t0 + L)
        sl = slice(t0, t1)
        blk = [np.ascontiguousarray(a[:, sl]) for a in (inp.q, inp.k, inp.v)]
        tabs = (inp.rope_cos[sl], inp.rope_sin[sl])
        before = state.copy()
        o0 = orc.step(*blk, *tabs, state, save=False)
        assert np.array_equal(state, before), "save=0 changed the state"
        o0b = orc.step(*blk, *tabs, state, save=False)
        assert np.array_equal(o0, o0b), "repeated save=0 steps differ"
        o1 = orc.step(*blk, *tabs, state, save=True)
        assert np.array_equal(o0, o1), "save flag changed the outputs"
        outs.append(o1)
    rows_close(np.concatenate(outs, axis=1), full, 1e-12, "step chain vs forward")
    assert np.abs(state - st_full).max() <= 1e-12 * np.abs(st_full).max(), "step state vs forward"
    # a non-zero initial state is added, not replaced
    st0 = np.random.default_rng(5).standard_normal((B, H, d + 1, d))
    st0[:, :, -1, :] = np.abs(st0[:, :, -1, :])
    outA, stA, _ = orc.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, N, 1e-8,
                                  state_in=st0)
    s = st0.copy()
    outB = orc.step(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, s, save=True)
    rows_close(outB, outA, 1e-12, "step vs recurrence with a carried state")
    _, st_local, _ = orc.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, N, 1e-8)
    assert np.abs(s - (st0 + st_local)).max() <= 1e-12 * np.abs(s).max(), "state = state_in + local"


def _exact_case(seed):
    rng = np.random.default_rng(seed)
    B, H, N, d = 1, 2, 7, 4
    q, k, v = (rng.integers(-8, 9, (B, N, H, d)) / 4.0 for _ in range(3))
    quarter = rng.integers(0, 4, (N, d // 2))
    cos = np.array([1, 0, -1, 0], np.float32)[quarter]
    sin = np.array([0, 1, 0, -1], np.float32)[quarter]
    return q.astype(np.float32), k.astype(np.float32), v.astype(np.float32), cos, sin


def _exact_reference(q, k, v, cos, sin, L, eps):
    B, N, H, d = q.shape
    F = Fraction
    out = np.empty(q.shape, np.float64)

    def rot(x, n):
        y = [F(0)] * d
        for p in range(d // 2):
            c, s = F(float(cos[n, p])), F(float(sin[n, p]))
            y[2 * p] = x[2 * p] * c - x[2 * p + 1] * s
            y[2 * p + 1] = x[2 * p] * s + x[2 * p + 1] * c
        return y

    for b in range(B):
        for h in range(H):
            fk = [[max(F(float(x)), F(0)) for x in k[b, j, h]] for j in range(N)]
            fq = [[max(F(float(x)), F(0)) for x in q[b, i, h]] for i in range(N)]
            for i in range(N):
                rq = rot(fq[i], i)
                num = [F(0)] * d
                den = F(eps)
                for j in range(N):
                    if j // L > i // L:
                        continue
                    a = sum(x * y for x, y in zip(rot(fk[j], j), rq))
                    for c in range(d):
                        num[c] += F(float(v[b, j, h, c])) * a
                    den += sum(x * y for x, y in zip(fk[j], fq[i]))
                for c in range(d):
                    out[b, i, h, c] = float(num[c] / den)
    return out


def pin_exact_rational(orc):
    """Dyadic inputs with quarter-turn rotary tables: the exact rational value
    of the definition, rounded once, within a few ulp."""
    eps = 2.0 ** -20
    for seed, L in [(41, 3), (42, 1), (43, 7), (44, 2)]:
        q, k, v, cos, sin = _exact_case(seed)
        ref = _exact_reference(q, k, v, cos, sin, L, eps)
        for route in ("masked", "recurrence"):
            if route == "masked":
                got = orc.masked(q, k, v, cos, sin, L, eps)
            else:
                got, _, _ = orc.recurrence(q, k, v, cos, sin, L, eps)
            rows_close(got, ref, 1e-14, f"exact rational {route} L={L}")


def pin_closed_forms(orc):
    """Single token: out = v a/(a + eps), a = phi(k).phi(q) (the rotation cancels
    at one position).  All-non-positive q row: out = 0 exactly.  Constant v with
    identity rotary and eps = 0: out = v.  eps enters the denominator once."""
    rng = np.random.default_rng(51)
    d = 8
    for trial in range(6):
        q, k, v = (rng.standard_normal((1, 1, 2, d)).astype(np.float32) for _ in range(3))
        if trial % 2 == 0:
            # quarter turns: the table entries are exact, the rotation cancels exactly
            quarter = rng.integers(0, 4, (1, d // 2))
            cos = np.array([1, 0, -1, 0], np.float32)[quarter]
            sin = np.array([0, 1, 0, -1], np.float32)[quarter]
            tol = 1e-13
        else:
            # float32 tables: cos^2 + sin^2 = 1 only to float32 rounding
            ang = rng.uniform(0, 2 * np.pi, (1, d // 2))
            cos, sin = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
            tol = 3e-7
        a = (np.maximum(q, 0).astype(np.float64) * np.maximum(k, 0)).sum(-1, keepdims=True)
        ref = v.astype(np.float64) * a / (a + 1e-8)
        for L in (1, 4):
            out, st, _ = orc.recurrence(q, k, v, cos, sin, L, 1e-8)
            rows_close(out, ref, tol, "single-token closed form")
            rows_close(orc.masked(q, k, v, cos, sin, L, 1e-8), ref, tol, "single-token masked")
    # non-positive q rows give exactly zero
    inp = small(52, N=19, d=8, L=4)
    q = inp.q.copy()
    q[:, 5] = -np.abs(q[:, 5])
    q[:, 11, 1] = 0.0
    for route in ("masked", "recurrence"):
        if route == "masked":
            o = orc.masked(q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, 4, 1e-8)
        else:
            o, _, _ = orc.recurrence(q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, 4, 1e-8)
        assert np.all(o[:, 5] == 0.0) and np.all(o[:, 11, 1] == 0.0), f"zero q row ({route})"
    # constant v, identity rotary, eps = 0 -> out = v wherever the denominator is positive
    inp = small(53, N=21, d=8, L=5)
    c = np.float32(1.25)
    v = np.full_like(inp.v, c)
    q = np.abs(inp.q) + np.float32(0.5)        # every row strictly positive
    k = np.abs(inp.k) + np.float32(0.5)
    ones = np.ones_like(inp.rope_cos)
    zeros = np.zeros_like(inp.rope_sin)
    for route in ("masked", "recurrence"):
        if route == "masked":
            o = orc.masked(q, k, v, ones, zeros, 5, 0.0)
        else:
            o, _, _ = orc.recurrence(q, k, v, ones, zeros, 5, 0.0)
        assert np.abs(o - 1.25).max() <= 1e-14, f"constant-v normalisation ({route})"
    # eps equal to the score halves the value: catches a dropped or misplaced eps
    q = np.zeros((1, 1, 1, d), np.float32)
    k = np.zeros((1, 1, 1, d), np.float32)
    q[..., 0] = 2.0 ** -14
    k[..., 0] = 2.0 ** -14
    v = rng.standard_normal((1, 1, 1, d)).astype(np.float32)
    cos = np.ones((1, d // 2), np.float32)
    sin = np.zeros((1, d // 2), np.float32)
    for route in ("masked", "recurrence"):
        if route == "masked":
            o = orc.masked(q, k, v, cos, sin, 1, 2.0 ** -28)
        else:
            o, _, _ = orc.recurrence(q, k, v, cos, sin, 1, 2.0 ** -28)
        assert np.array_equal(o, v.astype(np.float64) / 2), f"eps placement ({route})"


def pin_symmetries(orc):
    """Linearity in v; invariance under q -> alpha q (eps = 0); invariance under a
    shift of all positions (relative rotary); permuting tokens inside one block
    permutes only that block's outputs (bidirectional block); changing a block
    leaves earlier blocks alone and reaches every token of that block; the key
    sum z never decreases from block to block."""
    inp = small(61, B=1, H=2, N=30, d=8, L=7)
    q, k, v, c, s = inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin
    L = 7

    def run(q_, k_, v_, c_, s_, eps=1e-8):
        return orc.recurrence(q_, k_, v_, c_, s_, L, eps)[0]

    def run_m(q_, k_, v_, c_, s_, eps=1e-8):
        return orc.masked(q_, k_, v_, c_, s_, L, eps)

    rng = np.random.default_rng(62)
    # quarter-integer values so that 2 v1 - 3 v2 is exact in float32
    v1 = (rng.integers(-16, 17, v.shape) / 4.0).astype(np.float32)
    v2 = (rng.integers(-16, 17, v.shape) / 4.0).astype(np.float32)
    for f in (run, run_m):
        lhs = f(q, k, 2 * v1 - 3 * v2, c, s)
        rhs = 2 * f(q, k, v1, c, s) - 3 * f(q, k, v2, c, s)
        rows_close(lhs, rhs, 1e-12, "linearity in v")
        qd = (rng.integers(-16, 17, q.shape) / 4.0).astype(np.float32)
        rows_close(f(np.float32(0.75) * qd, k, v, c, s, 0.0), f(qd, k, v, c, s, 0.0), 1e-12,
                   "q scale invariance")
        # quarter-turn frequencies keep every table entry exact, so a shift of
        # all positions must leave the outputs unchanged to rounding
        m = np.array([0, 1, 2, 3])
        qc = np.array([1, 0, -1, 0], np.float32)
        qs = np.array([0, 1, 0, -1], np.float32)
        for shift in (1, 2, 7):
            n0 = np.arange(30)[:, None] * m[None, :] % 4
            n1 = (np.arange(30)[:, None] + shift) * m[None, :] % 4
            rows_close(f(q, k, v, qc[n1], qs[n1]), f(q, k, v, qc[n0], qs[n0]), 1e-12,
                       "position shift invariance (exact tables)")
        c1, s1 = rope_table_1d(30, 8, start=0)
        c2, s2 = rope_table_1d(30, 8, start=123)
        rows_close(f(q, k, v, c2, s2), f(q, k, v, c1, s1), 1e-5, "position shift invariance")
        # permutation inside block 1 (tokens 7..13) with its table rows
        perm = np.arange(30)
        perm[7:14] = 7 + rng.permutation(7)
        base = f(q, k, v, c, s)
        moved = f(q[:, perm], k[:, perm], v[:, perm], c[perm], s[perm])
        rows_close(moved, base[:, perm], 1e-12, "permutation inside a block")
        # perturb block 2 (tokens 14..20)
        k3 = k.copy()
        k3[:, 16] = np.abs(k3[:, 16]) + np.float32(1.0)
        v3 = v.copy()
        v3[:, 16] += np.float32(1.0)
        pert = f(q, k3, v3, c, s)
        assert np.array_equal(pert[:, :14], base[:, :14]), "earlier blocks changed"
        changed = np.abs(pert[:, 14:21] - base[:, 14:21]).max(axis=-1)
        fq = np.maximum(q[:, 14:21].astype(np.float64), 0).sum(-1)
        assert np.all(changed[fq > 0] > 0), "a token of the changed block did not see the change"
    _, _, pre = orc.recurrence(q, k, v, c, s, L, 1e-8, want_prefix=True)
    z = pre[:, :, :, -1, :]
    assert np.all(np.diff(z, axis=2) >= 0), "key sum decreased across blocks"


def pin_bf16_widening(orc):
    """bf16 bit patterns are read as their exact float32 values."""
    rng = np.random.default_rng(71)
    x = rng.standard_normal((1, 9, 2, 8)) * 3
    bits = [f64_to_bf16_bits(x * (i + 1)) for i in range(3)]
    wide = [bf16_bits_to_f32(b) for b in bits]
    c, s = rope_table_1d(9, 8)
    a, sa, _ = orc.recurrence(*bits, c, s, 4, 1e-8)
    b, sb, _ = orc.recurrence(*wide, c, s, 4, 1e-8)
    assert np.array_equal(a, b) and np.array_equal(sa, sb), "bf16 widening"
    ref = literal(*bits, c, s, 1e-8)
    rows_close(orc.recurrence(*bits, c, s, 9, 1e-8)[0], ref, 1e-12, "bf16 vs printed formula")


def masked_blocks_numpy(q, k, v, cos, sin, offsets, eps):
    """The definition pair by pair with an explicit block id per token:
    blk(n) = b for o[b] <= n < o[b+1]; token i takes every j with
    blk(j) <= blk(i).  Plain numpy, complex rotary; small N only."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    N = q.shape[1]
    blk = np.searchsorted(np.asarray(offsets), np.arange(N), side="right") - 1
    fq, fk = np.maximum(q, 0), np.maximum(k, 0)
    rq, rk = _complex_rotary(fq, cos, sin), _complex_rotary(fk, cos, sin)
    mask = (blk[None, :] <= blk[:, None]).astype(np.float64)          # [i, j]
    a = np.einsum("bihe,bjhe->bhij", rq, rk) * mask                    # rotated scores
    g = np.einsum("bihe,bjhe->bhij", fq, fk) * mask                    # normaliser terms
    num = np.einsum("bhij,bjhc->bihc", a, v)
    den = np.einsum("bhij->bih", g)[..., None] + eps
    return num / den


def pin_explicit_blocks(orc):
    """Explicit block boundaries (the blocks route, a step chain): random
    offsets with blocks of a single token, a first block one frame longer than
    the rest, and one block, against the pair-by-pair definition; uniform
    offsets against the block recurrence."""
    rng = np.random.default_rng(41)
    for seed, N, offs in [(41, 37, None), (42, 40, [0, 12, 20, 28, 36, 40]),   # 4 + 4k "frames" of 4
                          (43, 23, [0, 23]), (44, 30, [0, 1, 2, 3, 17, 18, 30])]:
        if offs is None:
            cuts = np.sort(rng.choice(np.arange(1, N), size=9, replace=False))
            offs = [0] + [int(c) for c in cuts] + [N]
        for dtype, dist in [("f32", "normal"), ("bf16", "laplace_negrows")]:
            inp = small(seed, N=N, d=8, dtype=dtype, dist=dist)
            out, st = orc.blocks(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, offs, 1e-8)
            ref = masked_blocks_numpy(inp.as_f32("q"), inp.as_f32("k"), inp.as_f32("v"),
                                      inp.rope_cos, inp.rope_sin, offs, 1e-8)
            rows_close(out, ref, 1e-12, f"blocks vs definition {offs}")
            # the final state is the sum over all tokens whatever the partition
            _, st1, _ = orc.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, N, 1e-8)
            assert np.abs(st - st1).max() <= 1e-12 * np.abs(st1).max(), "blocks state vs total"
    inp = small(45, N=33, d=8)
    L = 7
    offs = list(range(0, 33, L)) + [33]
    a, sa = orc.blocks(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, offs, 1e-8)
    b, sb, _ = orc.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, L, 1e-8)
    rows_close(a, b, 1e-12, "uniform offsets vs recurrence")


def pin_row_subset(orc):
    """Both routes evaluate a requested subset of rows (an unsorted list that
    spans several blocks, holds the first and last token and one repeat) into
    the slots in the order the rows were asked for.  Each row equals the same
    row of the full evaluation bit for bit, and the pair-by-pair definition
    written in numpy (explicit block ids, complex rotary) to 1e-12."""
    cases = [dict(seed=51, N=37, L=5, d=8, dtype="f32"),
             dict(seed=52, N=37, L=1, d=8, dtype="bf16", dist="laplace_negrows"),
             dict(seed=53, N=37, L=37, d=8, dtype="f32"),
             dict(seed=54, N=30, L=5, d=32, dtype="bf16"),
             dict(seed=55, N=26, L=1, d=32, dtype="f32"),
             dict(seed=56, N=22, L=22, d=64, dtype="bf16", dist="laplace_negrows"),
             dict(seed=57, N=22, L=5, d=64, dtype="f32")]
    for c in cases:
        N, L = c["N"], c["L"]
        inp = small(c["seed"], B=2, H=2, N=N, L=L, d=c["d"], dtype=c["dtype"],
                    dist=c.get("dist", "normal"))
        rng = np.random.default_rng(c["seed"])
        mid = rng.permutation(np.arange(1, N - 1))[: N // 3]
        rows = np.concatenate([[N - 1], mid[:2], [0], mid[2:], mid[:1]]).astype(np.int64)
        assert rows[0] > rows[1] or rows[1] > rows[2], "rows must be unsorted"
        args = (inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, L, 1e-8)
        full_m = orc.masked(*args)
        full_r, st_full, _ = orc.recurrence(*args)
        sub_m = orc.masked(*args, rows=rows)
        sub_r, st_sub, _ = orc.recurrence(*args, rows=rows)
        assert np.array_equal(sub_m, full_m[:, rows]), f"masked rows= vs full rows {c}"
        assert np.array_equal(sub_r, full_r[:, rows]), f"recurrence rows= vs full rows {c}"
        assert np.array_equal(st_sub, st_full), f"recurrence rows= changed the state {c}"
        offs = list(range(0, N, L)) + [N]
        ref = masked_blocks_numpy(inp.as_f32("q"), inp.as_f32("k"), inp.as_f32("v"),
                                  inp.rope_cos, inp.rope_sin, offs, 1e-8)[:, rows]
        rows_close(sub_m, ref, 1e-12, f"masked rows= vs definition {c}")
        rows_close(sub_r, ref, 1e-12, f"recurrence rows= vs definition {c}")


ALL_PINS = [pin_masked_equals_recurrence, pin_single_block_equals_printed_formula,
            pin_block_len_one_is_token_causal, pin_step_chain_equals_forward,
            pin_exact_rational, pin_closed_forms, pin_symmetries, pin_bf16_widening,
            pin_explicit_blocks, pin_row_subset]
