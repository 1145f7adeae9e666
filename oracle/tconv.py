"""fp64 oracle of the causal temporal convolution with a cached last frame.

TEST INFRASTRUCTURE, like the rest of ``oracle/``.

The pages say the causal Mix-FFN keeps the previous block's last frame for
its temporal convolution ("Block Causal Linear Attention", section "What
SANA-Video Actually Uses"; "[feat] LongSANA": causal computation for the
Mix-FFN, the convolution in the MLP) and give no kernel size.  With one frame
of history the convolution is read as depthwise, causal, of size 2 over latent
frames:

    y[b, f, s, c] = w[0, c] x[b, f, s, c] + w[1, c] x[b, f-1, s, c] + bias[c]

where frame -1 is the cache (zeros without one).  With save the cache becomes
the last frame of x.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

from workloads import bf16_bits_to_f32


def _widen(a: np.ndarray) -> np.ndarray:
    return (bf16_bits_to_f32(a) if a.dtype == np.uint16 else a).astype(np.float64)


def temporal_conv(x: np.ndarray, tokens_per_frame: int, weight: np.ndarray,
                  bias: Optional[np.ndarray] = None, cache: Optional[np.ndarray] = None
                  ) -> Tuple[np.ndarray, np.ndarray]:
    """x [B, F * S, C] (uint16 bf16 bits or float32), weight [2, C], bias [C]
    float32, cache [B, S, C] of x's type or None.  Returns (y [B, F * S, C]
    float64, the cache after saving: x's last frame, float64)."""
    xs = _widen(np.asarray(x))
    B, N, C = xs.shape
    S = int(tokens_per_frame)
    if S < 1 or N % S:
        raise ValueError("token count must be a whole number of frames")
    F = N // S
    frames = xs.reshape(B, F, S, C)
    prev = np.zeros((B, 1, S, C)) if cache is None else _widen(np.asarray(cache)).reshape(B, 1, S, C)
    shifted = np.concatenate([prev, frames[:, :-1]], axis=1)          # x[f - 1]
    w = np.asarray(weight, np.float64)
    b = np.zeros(C) if bias is None else np.asarray(bias, np.float64)
    y = w[0] * frames + w[1] * shifted + b
    last = frames[:, -1] if F > 0 else prev[:, 0]
    return y.reshape(B, N, C), last
