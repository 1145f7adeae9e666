"""The printed non-causal formula, written out in numpy (float64).

TEST INFRASTRUCTURE (see the package docstring for who may use it).

"Implementing Block Causal Linear Attention for Long Video Generation with
Sana", section "The Linear Attention Kernel", states the computation in the
channel-major layout (B, h, d, N):

    1. q, k, v reshaped to (B, h, d, N); ReLU applied to q and k;
    2. RoPE applied to the ReLU features (section "Rotary Position
       Embeddings") giving q_rotated, k_rotated;
    3. z = 1 / (k.sum(dim=-1, keepdim=True)^T @ q + eps)    (unrotated k, q)
       vk = v @ k_rotated^T
       out = vk @ q_rotated
       output = out * z

Summing over the whole sequence makes this the non-causal case, i.e. the
block-causal definition with a single block (block_len = N).  This module
follows those steps literally, with no blocking or reordering.
"""
from __future__ import annotations

import numpy as np


def _widen(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _rotary(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """x (B, h, d, N); cos/sin (N, d/2): rotate interleaved pairs (2p, 2p+1)."""
    c = cos.T.astype(np.float64)[None, None]          # (1, 1, d/2, N)
    s = sin.T.astype(np.float64)[None, None]
    a, b = x[:, :, 0::2, :], x[:, :, 1::2, :]
    y = np.empty_like(x)
    y[:, :, 0::2, :] = a * c - b * s
    y[:, :, 1::2, :] = a * s + b * c
    return y


def literal(q, k, v, rope_cos, rope_sin, eps: float = 1e-8) -> np.ndarray:
    """Non-causal output [B, N, H, d] following the printed steps."""
    # (B, N, H, d) -> (B, h, d, N)
    q = _widen(q).transpose(0, 2, 3, 1)
    k = _widen(k).transpose(0, 2, 3, 1)
    v = _widen(v).transpose(0, 2, 3, 1)
    q = np.maximum(q, 0.0)                            # kernel_func = ReLU
    k = np.maximum(k, 0.0)
    q_rotated = _rotary(q, rope_cos, rope_sin)
    k_rotated = _rotary(k, rope_cos, rope_sin)
    z = 1.0 / (np.swapaxes(k.sum(axis=-1, keepdims=True), -2, -1) @ q + eps)  # (B,h,1,N)
    vk = v @ np.swapaxes(k_rotated, -2, -1)           # (B, h, d, d)
    out = vk @ q_rotated                              # (B, h, d, N)
    output = out * z
    return output.transpose(0, 3, 1, 2)               # back to (B, N, h, d)
