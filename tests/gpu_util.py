"""Helpers for the GPU tests: move seeded inputs to the device and back."""
from __future__ import annotations

import numpy as np
import torch


def dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    """numpy (uint16 bf16 bits or float32) -> CUDA tensor of the same values."""
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def inputs_to_dev(inp, device="cuda"):
    return (dev(inp.q, device), dev(inp.k, device), dev(inp.v, device),
            dev(inp.rope_cos, device), dev(inp.rope_sin, device))


def host(t: torch.Tensor) -> np.ndarray:
    """CUDA tensor -> float64 numpy (exact for bf16 and fp32)."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def sample_rows(N: int, L: int, n: int, seed: int = 0) -> np.ndarray:
    """Random token indices plus the first and last token of every block and
    the last token of the sequence (block edges and the ragged tail)."""
    rng = np.random.default_rng(seed)
    nb = -(-N // L)
    edges = np.concatenate([np.arange(nb) * L, np.minimum(np.arange(1, nb + 1) * L, N) - 1])
    if len(edges) > 4 * n:
        edges = rng.choice(edges, 4 * n, replace=False)
    r = rng.choice(N, min(n, N), replace=False)
    return np.unique(np.concatenate([r, edges, [0, N - 1]]).astype(np.int64))
