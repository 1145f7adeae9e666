"""fp64 CPU oracle for block-causal ReLU linear attention.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the CUDA library and its binding) never imports it, and it never imports the
product path.

Routes (see ``lcla_oracle.c`` for the definition each one follows):
    masked(...)      the definition, pair by pair, O(N^2 d)
    recurrence(...)  per-block local states with a running inclusive sum
    step(...)        one block against a carried state, optional save
    blocks(...)      explicit block boundaries: the step route chained over the
                     blocks, each one saved into the carried state
    literal(...)     the printed non-causal formula (block_len = N), numpy

Inputs are numpy arrays: q, k, v [B, N, H, d] as uint16 bf16 bit patterns or
float32, rope tables [N, d/2] float32.  Results are float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

from .literal import literal  # noqa: F401  (numpy transcription)

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "lcla_oracle.c")
_SO = os.path.join(_HERE, "liblcla_oracle.so")


def compile_source(src: str, so: str) -> str:
    """gcc -O2 -fopenmp build of one oracle source file into a shared library."""
    tmp = so + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                           "-Wall", "-o", tmp, src])
    os.replace(tmp, so)
    return so


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liblcla_oracle.so`` when stale."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(SOURCE):
        compile_source(SOURCE, _SO)
    return _SO


class Oracle:
    """Handle on one build of the C oracle (the default build, or a test's)."""

    def __init__(self, so_path: Optional[str] = None):
        lib = ctypes.CDLL(so_path or build())
        P, I, D, L = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_int64
        lib.lcla_oracle_masked.argtypes = [P, P, P, I, P, P, I, I, I, I, I, D, P, L, P]
        lib.lcla_oracle_recurrence.argtypes = [P, P, P, I, P, P, I, I, I, I, I, D, P, P, L,
                                               P, P, P]
        lib.lcla_oracle_step.argtypes = [P, P, P, I, P, P, I, I, I, I, D, P, I, P]
        for f in (lib.lcla_oracle_masked, lib.lcla_oracle_recurrence, lib.lcla_oracle_step):
            f.restype = I
        lib.lcla_oracle_set_threads.argtypes = [I]
        lib.lcla_oracle_max_threads.restype = I
        self.lib = lib

    def set_threads(self, n: int) -> None:
        self.lib.lcla_oracle_set_threads(int(n))

    def max_threads(self) -> int:
        return int(self.lib.lcla_oracle_max_threads())

    def masked(self, q, k, v, rope_cos, rope_sin, block_len: int, eps: float = 1e-8,
               rows: Optional[np.ndarray] = None) -> np.ndarray:
        """Outputs [B, nrows, H, d] from the pair-by-pair definition."""
        q, k, v, c, s, code, (B, N, H, d) = _prep(q, k, v, rope_cos, rope_sin)
        r, nrows = _rows(rows, N)
        out = np.full((B, nrows, H, d), np.nan)     # a slot left unwritten stays NaN
        rc = self.lib.lcla_oracle_masked(_ptr(q), _ptr(k), _ptr(v), code, _ptr(c), _ptr(s),
                                         B, H, N, d, int(block_len), float(eps),
                                         _ptr(r), nrows, _ptr(out))
        if rc:
            raise ValueError("oracle masked: invalid argument")
        return out

    def recurrence(self, q, k, v, rope_cos, rope_sin, block_len: int, eps: float = 1e-8,
                   state_in: Optional[np.ndarray] = None, rows: Optional[np.ndarray] = None,
                   want_out: bool = True, want_prefix: bool = False):
        """Block-recurrence route.

        Returns (out [B, nrows, H, d] or None, state_out [B, H, d+1, d],
        prefix [B, H, nblocks, d+1, d] or None).
        """
        q, k, v, c, s, code, (B, N, H, d) = _prep(q, k, v, rope_cos, rope_sin)
        r, nrows = _rows(rows, N)
        if int(block_len) <= 0:
            raise ValueError("block_len must be positive")
        nb = -(-N // int(block_len))
        out = np.full((B, nrows, H, d), np.nan) if want_out else None   # unwritten slots stay NaN
        st = np.empty((B, H, d + 1, d), np.float64)
        pre = np.empty((B, H, nb, d + 1, d), np.float64) if want_prefix else None
        sin_ = None
        if state_in is not None:
            sin_ = np.ascontiguousarray(state_in, dtype=np.float64)
            if sin_.shape != (B, H, d + 1, d):
                raise ValueError("state_in must be [B, H, d+1, d]")
        rc = self.lib.lcla_oracle_recurrence(_ptr(q), _ptr(k), _ptr(v), code, _ptr(c), _ptr(s),
                                             B, H, N, d, int(block_len), float(eps), _ptr(sin_),
                                             _ptr(r), nrows, _ptr(out), _ptr(st), _ptr(pre))
        if rc:
            raise ValueError("oracle recurrence: invalid argument")
        return out, st, pre

    def step(self, q, k, v, rope_cos, rope_sin, state: np.ndarray, save: bool,
             eps: float = 1e-8) -> np.ndarray:
        """One block against ``state`` (float64 [B, H, d+1, d], updated in place
        when ``save``).  Returns the block's outputs [B, L, H, d]."""
        q, k, v, c, s, code, (B, L, H, d) = _prep(q, k, v, rope_cos, rope_sin)
        if (state.dtype != np.float64 or not state.flags.c_contiguous
                or state.shape != (B, H, d + 1, d)):
            raise ValueError("state must be C-contiguous float64 [B, H, d+1, d]")
        out = np.empty((B, L, H, d), np.float64)
        rc = self.lib.lcla_oracle_step(_ptr(q), _ptr(k), _ptr(v), code, _ptr(c), _ptr(s),
                                       B, H, L, d, float(eps), _ptr(state), int(bool(save)),
                                       _ptr(out))
        if rc:
            raise ValueError("oracle step: invalid argument")
        return out


    def blocks(self, q, k, v, rope_cos, rope_sin, offsets, eps: float = 1e-8,
               state_in: Optional[np.ndarray] = None):
        """Block boundaries given as token offsets 0 = o[0] < ... < o[nb] = N:
        block b is [o[b], o[b+1]) and attends to itself and every earlier
        block, which is the step route run block after block with save.
        Returns (out [B, N, H, d], state_out [B, H, d+1, d]), float64."""
        q = np.ascontiguousarray(q)
        B, N, H, d = q.shape
        o = [int(x) for x in np.asarray(offsets).ravel()]
        if len(o) < 2 or o[0] != 0 or o[-1] != N or any(b <= a for a, b in zip(o, o[1:])):
            raise ValueError("offsets must rise strictly from 0 to N")
        state = np.zeros((B, H, d + 1, d), np.float64) if state_in is None else \
            np.array(state_in, dtype=np.float64, order="C", copy=True)
        out = np.empty((B, N, H, d), np.float64)
        for a, b in zip(o, o[1:]):
            out[:, a:b] = self.step(q[:, a:b], np.asarray(k)[:, a:b], np.asarray(v)[:, a:b],
                                    np.asarray(rope_cos)[a:b], np.asarray(rope_sin)[a:b], state, True, eps)
        return out, state


_default: Optional[Oracle] = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def set_threads(n: int) -> None:
    default().set_threads(n)


def max_threads() -> int:
    return default().max_threads()


def masked(*a, **kw):
    return default().masked(*a, **kw)


def recurrence(*a, **kw):
    return default().recurrence(*a, **kw)


def step(*a, **kw):
    return default().step(*a, **kw)


def blocks(*a, **kw):
    return default().blocks(*a, **kw)


def _prep(q, k, v, rope_cos, rope_sin):
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    if not (q.dtype == k.dtype == v.dtype) or q.dtype not in (np.uint16, np.float32):
        raise TypeError("q, k, v must all be uint16 (bf16 bits) or all float32")
    if not (q.shape == k.shape == v.shape) or q.ndim != 4:
        raise ValueError("q, k, v must share one [B, N, H, d] shape")
    B, N, H, d = q.shape
    c = np.ascontiguousarray(rope_cos, dtype=np.float32)
    s = np.ascontiguousarray(rope_sin, dtype=np.float32)
    if c.shape != (N, d // 2) or s.shape != (N, d // 2):
        raise ValueError("rope tables must be [N, d/2]")
    code = 0 if q.dtype == np.uint16 else 1
    return q, k, v, c, s, code, (B, N, H, d)


def _ptr(a):
    return None if a is None else a.ctypes.data


def _rows(rows, N):
    if rows is None:
        return None, N
    r = np.ascontiguousarray(rows, dtype=np.int64)
    return r, len(r)
