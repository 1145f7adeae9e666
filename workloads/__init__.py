"""Seeded synthetic inputs for block-causal ReLU linear attention.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests. It holds none of the attention method's arithmetic: it draws
q, k, v from the stated distributions, rounds them to the storage dtype
(round-to-nearest-even), and builds the rotary-embedding cos/sin tables that a
caller passes to the library as plain inputs (the library only applies them).

Array conventions
-----------------
* q, k, v: layout [B, N, H, d], C order.  bf16 tensors are returned as their
  raw ``uint16`` bit patterns, fp32 tensors as ``float32``.  ``as_f32`` widens
  bf16 bits exactly.
* rope_cos, rope_sin: ``float32`` [N, d/2]; pair p of a token rotates the
  interleaved elements (2p, 2p+1) of that token's head vector.  Frequencies
  follow the usual rotary form theta**(-2j/D) per axis of D dims.

Distributions (one row = the d values of one (b, n, h)):
* ``normal``: N(0, sigma^2) elementwise.
* ``laplace_negrows``: Laplace(0, 1) elementwise, then every row independently
  with probability 0.3 replaced by ``-|row|`` (all entries <= 0, so the ReLU
  feature map sends it to zero).
"""
from __future__ import annotations

import os
import threading
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace
from typing import Optional, Tuple

import numpy as np

__all__ = [
    "f64_to_bf16_bits", "bf16_bits_to_f32", "rope_table_1d", "rope_table_3d",
    "Spec", "Inputs", "make_inputs", "named", "NAMED",
]

_CHUNK = 1 << 22          # elements per independently seeded chunk (multiple of d)
_NEG_ROW_P = 0.3          # share of rows forced entirely non-positive


# ----------------------------------------------------------------------------
# rounding helpers
# ----------------------------------------------------------------------------
def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (nearest, ties to even); return uint16 bits.

    Rounds once, directly from float64 (no intermediate float32 rounding), by
    clearing the 45 low mantissa bits of the binary64 pattern with a
    round-half-even carry.  The result then has at most 8 significant bits, so
    its float32 image is exact and bf16 is that image's top half.  Values in
    the bf16 subnormal range are rejected (the distributions here never
    produce them).
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite sample")
    ax = np.abs(x)
    if np.any((ax < 2.0 ** -126) & (ax != 0.0)):
        raise ValueError("sample in the bf16 subnormal range")
    b = x.view(np.uint64)
    lsb = (b >> np.uint64(45)) & np.uint64(1)
    b = (b + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    f = b.view(np.float64).astype(np.float32)
    if not np.all(np.isfinite(f)):
        raise ValueError("sample overflows bf16")
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    u = np.ascontiguousarray(u, dtype=np.uint16)
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------
# rotary tables (inputs of the method, built the usual way)
# ----------------------------------------------------------------------------
def _inv_freq(D: int, theta: float) -> np.ndarray:
    return theta ** (-(2.0 * np.arange(D // 2, dtype=np.float64)) / D)


def rope_table_1d(N: int, d: int = 32, theta: float = 10000.0,
                  start: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """cos/sin [N, d/2] float32 for positions start..start+N-1 over all d dims."""
    pos = np.arange(start, start + N, dtype=np.float64)[:, None]
    ang = pos * _inv_freq(d, theta)[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def rope_table_3d(frames: int, Hg: int, Wg: int, dims=(8, 12, 12),
                  theta: float = 10000.0, frame_start: int = 0
                  ) -> Tuple[np.ndarray, np.ndarray]:
    """cos/sin [frames*Hg*Wg, sum(dims)/2] float32 for a (t, h, w) token grid.

    Token order is n = f*(Hg*Wg) + r*Wg + c.  The first dims[0]/2 pairs carry
    the frame index (absolute: frame_start + f), the next dims[1]/2 the row,
    the last dims[2]/2 the column; each axis uses its own theta**(-2j/D_axis).
    """
    f = np.arange(frame_start, frame_start + frames, dtype=np.float64)
    r = np.arange(Hg, dtype=np.float64)
    c = np.arange(Wg, dtype=np.float64)
    F, R, C = np.meshgrid(f, r, c, indexing="ij")
    parts = []
    for coord, D in zip((F.ravel(), R.ravel(), C.ravel()), dims):
        parts.append(coord[:, None] * _inv_freq(D, theta)[None, :])
    ang = np.concatenate(parts, axis=1)
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


# ----------------------------------------------------------------------------
# workload specification and generation
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class Spec:
    """Shape, dtype, distribution and seed of one synthetic workload."""
    name: str
    B: int
    H: int
    N: int
    d: int
    block_len: int
    dtype: str                    # "bf16" or "f32"
    seed: int
    qk_dist: str = "normal"       # "normal" or "laplace_negrows"
    v_sigma: float = 1.0
    rope: str = "1d"              # "1d" or "3d"
    grid: Optional[Tuple[int, int, int]] = None   # (frames, Hg, Wg) for 3d
    eps: float = 1e-8
    theta: float = 10000.0

    @property
    def nblocks(self) -> int:
        return -(-self.N // self.block_len)

    @property
    def token_heads(self) -> int:
        return self.B * self.N * self.H

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4


@dataclass
class Inputs:
    spec: Spec
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    rope_cos: np.ndarray
    rope_sin: np.ndarray
    extra: dict = field(default_factory=dict)

    def as_f32(self, name: str) -> np.ndarray:
        a = getattr(self, name)
        return bf16_bits_to_f32(a) if a.dtype == np.uint16 else a


def _seed_seq(seed: int, tensor_id: int, chunk: int) -> np.random.SeedSequence:
    return np.random.SeedSequence(entropy=seed, spawn_key=(tensor_id, chunk))


_scratch = threading.local()


def _buffers(n: int):
    """This thread's reusable chunk buffers (float64, uint64, float32, uint32).
    Reusing them keeps the threads off the allocator: fresh chunk-sized
    arrays are mapped and unmapped per call, and the page faults and
    unmappings serialise the threads."""
    bufs = getattr(_scratch, "bufs", None)
    if bufs is None or bufs[0].size < n:
        bufs = (np.empty(n, np.float64), np.empty(n, np.uint64), np.empty(n, np.float32),
                np.empty(n, np.uint32))
        _scratch.bufs = bufs
    return tuple(b[:n] for b in bufs)


def _round_bf16_into(x: np.ndarray, t64: np.ndarray, f32: np.ndarray, u32: np.ndarray,
                     out: np.ndarray):
    """``f64_to_bf16_bits(x)`` written into ``out`` (uint16) through the
    caller's buffers; ``x`` is overwritten.  The same checks and bits."""
    ax = np.abs(x, out=t64.view(np.float64))
    if not np.isfinite(ax.max()):
        raise ValueError("non-finite sample")
    if np.count_nonzero(ax < 2.0 ** -126) != np.count_nonzero(ax == 0.0):
        raise ValueError("sample in the bf16 subnormal range")
    b = x.view(np.uint64)
    np.right_shift(b, np.uint64(45), out=t64)
    np.bitwise_and(t64, np.uint64(1), out=t64)
    np.add(t64, np.uint64((1 << 44) - 1), out=t64)
    np.add(b, t64, out=b)
    np.bitwise_and(b, ~np.uint64((1 << 45) - 1), out=b)
    f32[:] = x
    if not np.isfinite(np.abs(f32).max()):
        raise ValueError("sample overflows bf16")
    np.right_shift(f32.view(np.uint32), np.uint32(16), out=u32)
    out[:] = u32


def _fill_chunk(out: np.ndarray, lo: int, hi: int, d: int, seed: int,
                tensor_id: int, chunk: int, dist: str, sigma: float, dtype: str):
    rng = np.random.Generator(np.random.PCG64(_seed_seq(seed, tensor_id, chunk)))
    n = hi - lo
    x, t64, f32, u32 = _buffers(n)
    if dist == "normal":
        rng.standard_normal(out=x)
        x *= sigma
    elif dist == "laplace_negrows":
        x[:] = rng.laplace(0.0, 1.0, n)
        rows = x.reshape(-1, d)
        neg = rng.random(rows.shape[0]) < _NEG_ROW_P
        rows[neg] = -np.abs(rows[neg])
    else:
        raise ValueError(dist)
    if dtype == "bf16":
        _round_bf16_into(x, t64, f32, u32, out[lo:hi])
    else:
        out[lo:hi] = x


def _draw_tensor(shape, d: int, seed: int, tensor_id: int, dist: str,
                 sigma: float, dtype: str, threads: Optional[int] = None):
    total = int(np.prod(shape))
    assert _CHUNK % d == 0
    out = np.empty(total, dtype=np.uint16 if dtype == "bf16" else np.float32)
    bounds = [(lo, min(lo + _CHUNK, total)) for lo in range(0, total, _CHUNK)]
    threads = threads or min(len(bounds), os.cpu_count() or 1)
    if threads <= 1:
        for i, (lo, hi) in enumerate(bounds):
            _fill_chunk(out, lo, hi, d, seed, tensor_id, i, dist, sigma, dtype)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda a: _fill_chunk(out, a[1][0], a[1][1], d, seed,
                                              tensor_id, a[0], dist, sigma, dtype),
                        enumerate(bounds)))
    return out.reshape(shape)


def make_tables(spec: Spec, start_token: int = 0, count: Optional[int] = None):
    """RoPE tables for tokens [start_token, start_token+count) of ``spec``."""
    count = spec.N - start_token if count is None else count
    if spec.rope == "1d":
        return rope_table_1d(count, spec.d, spec.theta, start=start_token)
    frames, Hg, Wg = spec.grid
    per = Hg * Wg
    f0 = start_token // per
    f1 = -(-(start_token + count) // per)
    c, s = rope_table_3d(f1 - f0, Hg, Wg, theta=spec.theta, frame_start=f0,
                         dims=_dims3d(spec.d))
    off = start_token - f0 * per
    return (np.ascontiguousarray(c[off:off + count]),
            np.ascontiguousarray(s[off:off + count]))


def _dims3d(d: int):
    if d == 32:
        return (8, 12, 12)
    if d == 64:
        return (16, 24, 24)
    raise ValueError("3D rotary split defined for d in {32, 64}")


def make_inputs(spec: Spec, threads: Optional[int] = None) -> Inputs:
    """Draw q, k, v and build the tables for ``spec`` (deterministic in seed)."""
    shape = (spec.B, spec.N, spec.H, spec.d)
    q = _draw_tensor(shape, spec.d, spec.seed, 0, spec.qk_dist, 1.0, spec.dtype, threads)
    k = _draw_tensor(shape, spec.d, spec.seed, 1, spec.qk_dist, 1.0, spec.dtype, threads)
    v = _draw_tensor(shape, spec.d, spec.seed, 2, "normal", spec.v_sigma, spec.dtype, threads)
    c, s = make_tables(spec)
    return Inputs(spec, q, k, v, c, s)


def _robust(dtype: str, L: int, seed: int) -> Spec:
    return Spec(f"robust_{dtype}_L{L}", 1, 16, 65536, 32, L, dtype, seed,
                qk_dist="laplace_negrows", v_sigma=2.0, rope="1d")


# The named workloads: tiny parity case, 480p-like forward, streaming blocks,
# minute-scale forward, the 480p-like forward at head dim 64, and the
# robustness sweep over block lengths.
NAMED = {
    "tiny_f32": Spec("tiny_f32", 1, 2, 1024, 32, 256, "f32", 0),
    "fwd480p_bf16": Spec("fwd480p_bf16", 1, 70, 21 * 30 * 52, 32, 3 * 30 * 52, "bf16", 1,
                         rope="3d", grid=(21, 30, 52)),
    "stream_bf16": Spec("stream_bf16", 2, 70, 41 * 30 * 52, 32, 3 * 30 * 52, "bf16", 2,
                        rope="3d", grid=(41, 30, 52)),
    "minute_bf16": Spec("minute_bf16", 1, 70, 241 * 44 * 80, 32, 3 * 44 * 80, "bf16", 3,
                        rope="3d", grid=(241, 44, 80)),
    # linear_head_dim 64 at the same model width (35 heads x 64 = 2240)
    "fwd480p_d64_bf16": Spec("fwd480p_d64_bf16", 1, 35, 21 * 30 * 52, 64, 3 * 30 * 52, "bf16", 12,
                             rope="3d", grid=(21, 30, 52)),
    # the same latent with fp32 inputs (the CUDA-core head-dim-64 passes)
    "fwd480p_d64_f32": Spec("fwd480p_d64_f32", 1, 35, 21 * 30 * 52, 64, 3 * 30 * 52, "f32", 13,
                            rope="3d", grid=(21, 30, 52)),
}
for _i, _L in enumerate((1, 64, 1560, 4680, 65536)):
    for _dt in ("f32", "bf16"):
        NAMED[f"robust_{_dt}_L{_L}"] = _robust(_dt, _L, 4 + _i)


def named(name: str, **overrides) -> Spec:
    spec = NAMED[name]
    return replace(spec, **overrides) if overrides else spec
