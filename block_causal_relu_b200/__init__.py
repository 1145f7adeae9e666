"""Block-causal ReLU linear attention with a carried fp32 state, on B200.

Thin binding of the C-ABI library ``liblcla.so`` (declared in
``include/lcla.h``): it checks and marshals torch tensors (device memory and
the current CUDA stream) into its entry points -- the whole-sequence forward
(uniform or explicit blocks), the streaming step, the two halves of a
sequence-sharded forward and the Mix-FFN temporal convolution.  Every step of
the computation runs in the library's sm_100a kernels; there is no other path.
Importing this package fails if the library has not been built
(``python block_causal_relu_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

__all__ = ["forward", "step", "forward_workspace_bytes", "step_workspace_bytes", "plan_info",
           "forward_blocks", "forward_blocks_workspace_bytes", "temporal_conv",
           "shard_begin", "shard_end", "shard_workspace_bytes", "device_status", "selftest_bounded_wait",
           "LclaError", "LIB_PATH", "lib", "BF16", "F32", "D", "HEAD_DIMS"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblcla.so")
BF16, F32 = 0, 1
D = 32                 # head dim of the tensor-core path
HEAD_DIMS = (32, 64)   # head dims the library serves
DEFAULT_EPS = 1e-8


class LclaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"lcla status {status}: {msg}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python block_causal_relu_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.lcla_forward_workspace_bytes.argtypes = [I, I, I, I, I, I]
    L.lcla_forward_workspace_bytes.restype = Z
    L.lcla_step_workspace_bytes.argtypes = [I, I, I, I, I]
    L.lcla_step_workspace_bytes.restype = Z
    L.lcla_forward.argtypes = [P, P, P, P, P, I, I, I, I, I, F, P, P, I, P, Z, P]
    L.lcla_forward.restype = I
    L.lcla_forward_timed.argtypes = [P, P, P, P, P, I, I, I, I, I, F, P, P, I, P, Z, P, P]
    L.lcla_forward_timed.restype = I
    L.lcla_step.argtypes = [P, P, P, P, P, I, I, I, I, F, P, I, P, I, P, Z, P]
    L.lcla_step.restype = I
    L.lcla_forward_blocks_workspace_bytes.argtypes = [I, I, I, I, I, I]
    L.lcla_forward_blocks_workspace_bytes.restype = Z
    L.lcla_forward_blocks.argtypes = [P, P, P, P, P, I, I, I, I, P, I, F, P, P, I, P, Z, P]
    L.lcla_forward_blocks.restype = I
    L.lcla_temporal_conv.argtypes = [P, I, I, I, I, P, P, P, I, P, I, P]
    L.lcla_temporal_conv.restype = I
    L.lcla_shard_workspace_bytes.argtypes = [I, I, I, I, I, I]
    L.lcla_shard_workspace_bytes.restype = Z
    L.lcla_shard_begin.argtypes = [P, P, P, P, I, I, I, I, I, P, I, P, Z, P]
    L.lcla_shard_begin.restype = I
    L.lcla_shard_end.argtypes = [P, P, P, P, P, I, I, I, I, I, F, P, I, I, P, P, P, I, P, Z, P]
    L.lcla_shard_end.restype = I
    L.lcla_selftest_bounded_wait.argtypes = [I, P, P]
    L.lcla_selftest_bounded_wait.restype = I
    L.lcla_forward_plan_info.argtypes = [I, I, I, I, I, I, P]
    L.lcla_forward_plan_segments.argtypes = [I, I, I, I, I, I, P, P, P, I]
    L.lcla_forward_plan_segments.restype = I
    L.lcla_forward_plan_info.restype = I
    L.lcla_status_string.argtypes = [I]
    L.lcla_status_string.restype = ctypes.c_char_p
    L.lcla_version.restype = I
    return L


lib = _load()


def _check(rc: int) -> None:
    if rc != 0:
        raise LclaError(rc, lib.lcla_status_string(rc).decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"q, k, v must be bfloat16 or float32, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _inputs(q, k, v, cos, sin):
    for name, t in (("q", q), ("k", k), ("v", v), ("cos", cos), ("sin", sin)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one [B, N, H, d] shape")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    B, N, H, d = q.shape
    if cos.dtype != torch.float32 or sin.dtype != torch.float32:
        raise TypeError("rope tables must be float32")
    if tuple(cos.shape) != (N, d // 2) or tuple(sin.shape) != (N, d // 2):
        raise ValueError("rope tables must be [N, d/2]")
    return B, N, H, d, _dtype_code(q)


def forward_workspace_bytes(B: int, H: int, N: int, d: int, block_len: int, dtype: int) -> int:
    return int(lib.lcla_forward_workspace_bytes(B, H, N, d, block_len, dtype))


def forward_blocks_workspace_bytes(B: int, H: int, N: int, d: int, nblocks: int, dtype: int) -> int:
    return int(lib.lcla_forward_blocks_workspace_bytes(B, H, N, d, nblocks, dtype))


def step_workspace_bytes(B: int, H: int, L: int, d: int, dtype: int) -> int:
    return int(lib.lcla_step_workspace_bytes(B, H, L, d, dtype))


def plan_info(B: int, H: int, N: int, d: int, block_len: int, dtype: int) -> dict:
    """The library's cut of a forward problem (see ``lcla_forward_plan_info``)."""
    info = (ctypes.c_int * 5)()
    _check(lib.lcla_forward_plan_info(B, H, N, d, block_len, dtype, info))
    return {"chunk_mode": bool(info[0]), "segments": info[1], "prefixes": info[2],
            "tile_tokens": info[3], "tensor_cores": bool(info[4])}


def plan_segments(B: int, H: int, N: int, d: int, block_len: int, dtype: int) -> list:
    """``lcla_forward_plan_segments``: [(t0, t1, block or -1), ...] per segment."""
    n = plan_info(B, H, N, d, block_len, dtype)["segments"]
    arr = [(ctypes.c_int * max(n, 1))() for _ in range(3)]
    _check(lib.lcla_forward_plan_segments(B, H, N, d, block_len, dtype, arr[0], arr[1], arr[2], n))
    return [(arr[0][i], arr[1][i], arr[2][i]) for i in range(n)]


def _stream(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else int(stream)


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rope_cos: torch.Tensor,
            rope_sin: torch.Tensor, block_len: int, eps: float = DEFAULT_EPS, *,
            out: Optional[torch.Tensor] = None, state_out: Optional[torch.Tensor] = None,
            want_state: bool = True, workspace: Optional[torch.Tensor] = None,
            stream=None, events=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """``lcla_forward``: whole-sequence block-causal attention.

    q, k, v [B, N, H, d] (bf16 or fp32), rope tables [N, d/2] fp32, all CUDA.
    Returns (out [B, N, H, d], state_out [B, H, d+1, d] fp32 or None).
    Buffers not passed in are allocated with torch on q's device.
    ``events``: optional 4 already-recorded ``torch.cuda.Event(enable_timing=True)``
    that the library re-records around its passes (``lcla_forward_timed``).
    """
    B, N, H, d, code = _inputs(q, k, v, rope_cos, rope_sin)
    if out is None:
        out = torch.empty_like(q)
    if state_out is None and want_state:
        state_out = torch.empty((B, H, d + 1, d), dtype=torch.float32, device=q.device)
    need = forward_workspace_bytes(B, H, N, d, block_len, code)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    evp = None
    if events is not None:
        if len(events) != 4:
            raise ValueError("events must hold 4 torch.cuda.Event")
        evp = (ctypes.c_void_p * 4)(*[e.cuda_event for e in events])
    _check(lib.lcla_forward_timed(_ptr(q), _ptr(k), _ptr(v), _ptr(rope_cos), _ptr(rope_sin),
                                  B, H, N, d, int(block_len), float(eps), _ptr(out),
                                  _ptr(state_out), code, _ptr(workspace),
                                  0 if workspace is None else workspace.numel(),
                                  _stream(stream, q.device), evp))
    return out, state_out


def forward_blocks(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rope_cos: torch.Tensor,
                   rope_sin: torch.Tensor, block_offsets: torch.Tensor, eps: float = DEFAULT_EPS, *,
                   out: Optional[torch.Tensor] = None, state_out: Optional[torch.Tensor] = None,
                   want_state: bool = True, workspace: Optional[torch.Tensor] = None,
                   stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """``lcla_forward_blocks``: as ``forward`` with explicit block boundaries,
    ``block_offsets`` an int32 CUDA tensor [nblocks + 1] rising from 0 to N."""
    B, N, H, d, code = _inputs(q, k, v, rope_cos, rope_sin)
    if (not isinstance(block_offsets, torch.Tensor) or not block_offsets.is_cuda
            or block_offsets.dtype != torch.int32 or block_offsets.dim() != 1
            or not block_offsets.is_contiguous()):
        raise ValueError("block_offsets must be a contiguous int32 CUDA tensor [nblocks + 1]")
    nblocks = block_offsets.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    if state_out is None and want_state:
        state_out = torch.empty((B, H, d + 1, d), dtype=torch.float32, device=q.device)
    need = forward_blocks_workspace_bytes(B, H, N, d, nblocks, code)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check(lib.lcla_forward_blocks(_ptr(q), _ptr(k), _ptr(v), _ptr(rope_cos), _ptr(rope_sin),
                                   B, H, N, d, _ptr(block_offsets), nblocks, float(eps), _ptr(out),
                                   _ptr(state_out), code, _ptr(workspace),
                                   0 if workspace is None else workspace.numel(),
                                   _stream(stream, q.device)))
    return out, state_out


def shard_workspace_bytes(B: int, H: int, N: int, d: int, block_len: int, dtype: int) -> int:
    return int(lib.lcla_shard_workspace_bytes(B, H, N, d, block_len, dtype))


def _state_tensor(name: str, t: Optional[torch.Tensor], B: int, H: int, d: int, lead=()) -> None:
    if t is None:
        return
    if (not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.float32
            or not t.is_contiguous() or tuple(t.shape) != (*lead, B, H, d + 1, d)):
        raise ValueError(f"{name} must be a contiguous float32 CUDA tensor {[*lead, B, H, d + 1, d]}")


def shard_begin(k: torch.Tensor, v: torch.Tensor, rope_cos: torch.Tensor, rope_sin: torch.Tensor,
                block_len: int, *, total_out: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None,
                stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """``lcla_shard_begin``: this rank's state total over its tokens k, v
    [B, N, H, d] (whole blocks of the sequence, tables at their absolute
    positions).  Returns (total [B, H, d+1, d] fp32, workspace); pass the same
    workspace to ``shard_end``."""
    B, N, H, d, code = _inputs(k, k, v, rope_cos, rope_sin)
    if total_out is None:
        total_out = torch.empty((B, H, d + 1, d), dtype=torch.float32, device=k.device)
    _state_tensor("total_out", total_out, B, H, d)
    need = shard_workspace_bytes(B, H, N, d, block_len, code)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=k.device)
    _check(lib.lcla_shard_begin(_ptr(k), _ptr(v), _ptr(rope_cos), _ptr(rope_sin), B, H, N, d, int(block_len),
                                _ptr(total_out), code, _ptr(workspace),
                                0 if workspace is None else workspace.numel(), _stream(stream, k.device)))
    return total_out, workspace


def shard_end(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rope_cos: torch.Tensor,
              rope_sin: torch.Tensor, block_len: int, totals: torch.Tensor, rank: int,
              workspace: Optional[torch.Tensor], eps: float = DEFAULT_EPS, *,
              state_in: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
              state_out: Optional[torch.Tensor] = None, want_state: bool = True,
              stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """``lcla_shard_end``: this rank's outputs from the gathered ``totals``
    [R, B, H, d+1, d] (every rank's ``shard_begin`` total, in rank order) and
    the workspace ``shard_begin`` filled.  Returns (out, state after the whole
    sequence, or None)."""
    B, N, H, d, code = _inputs(q, k, v, rope_cos, rope_sin)
    if not isinstance(totals, torch.Tensor) or totals.dim() != 5:
        raise ValueError("totals must be [R, B, H, d+1, d]")
    nranks = totals.shape[0]
    _state_tensor("totals", totals, B, H, d, lead=(nranks,))
    _state_tensor("state_in", state_in, B, H, d)
    if out is None:
        out = torch.empty_like(q)
    if state_out is None and want_state:
        state_out = torch.empty((B, H, d + 1, d), dtype=torch.float32, device=q.device)
    _state_tensor("state_out", state_out, B, H, d)
    _check(lib.lcla_shard_end(_ptr(q), _ptr(k), _ptr(v), _ptr(rope_cos), _ptr(rope_sin), B, H, N, d,
                              int(block_len), float(eps), _ptr(totals), nranks, int(rank), _ptr(state_in),
                              _ptr(out), _ptr(state_out), code, _ptr(workspace),
                              0 if workspace is None else workspace.numel(), _stream(stream, q.device)))
    return out, state_out


def device_status(workspace: Optional[torch.Tensor]) -> int:
    """The device status word a call left in ``workspace`` (0: every bounded
    wait completed; bit 0 / bit 1: pass A / pass C gave up).  Synchronises on
    the copy."""
    if workspace is None or workspace.numel() < 4:
        return 0
    return int(workspace[:4].view(torch.int32).item())


def selftest_bounded_wait(arrive_first: bool, stream=None) -> Tuple[bool, int, int]:
    """``lcla_selftest_bounded_wait``: (gave_up, nanoseconds waited, abort flag)."""
    res = torch.zeros(3, dtype=torch.int64, device="cuda")
    _check(lib.lcla_selftest_bounded_wait(int(bool(arrive_first)), _ptr(res), _stream(stream, res.device)))
    r = res.cpu().tolist()
    return bool(r[0]), int(r[1]), int(r[2])


def step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cos: torch.Tensor,
         sin: torch.Tensor, state: torch.Tensor, save: bool, eps: float = DEFAULT_EPS, *,
         out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
         stream=None) -> torch.Tensor:
    """``lcla_step``: one block [B, L, H, d] against ``state`` [B, H, d+1, d]
    fp32 (updated in place when ``save``).  Returns the block's outputs."""
    B, L, H, d, code = _inputs(q, k, v, cos, sin)
    if (not state.is_cuda or state.dtype != torch.float32 or not state.is_contiguous()
            or tuple(state.shape) != (B, H, d + 1, d)):
        raise ValueError("state must be a contiguous float32 CUDA tensor [B, H, d+1, d]")
    if out is None:
        out = torch.empty_like(q)
    need = step_workspace_bytes(B, H, L, d, code)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check(lib.lcla_step(_ptr(q), _ptr(k), _ptr(v), _ptr(cos), _ptr(sin), B, H, L, d, float(eps),
                         _ptr(state), int(bool(save)), _ptr(out), code, _ptr(workspace),
                         0 if workspace is None else workspace.numel(), _stream(stream, q.device)))
    return out


def temporal_conv(x: torch.Tensor, tokens_per_frame: int, weight: torch.Tensor,
                  bias: Optional[torch.Tensor] = None, cache: Optional[torch.Tensor] = None,
                  save: bool = False, *, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """``lcla_temporal_conv``: causal size-2 depthwise convolution over latent
    frames of ``x`` [B, F * S, C] (S = ``tokens_per_frame``), with weight [2, C]
    and bias [C] fp32 and the previous frame from ``cache`` [B, S, C] (zeros
    when None); ``save`` overwrites the cache with x's last frame."""
    if not isinstance(x, torch.Tensor) or not x.is_cuda or not x.is_contiguous() or x.dim() != 3:
        raise ValueError("x must be a contiguous CUDA tensor [B, F * S, C]")
    B, N, C = x.shape
    S = int(tokens_per_frame)
    if S < 1 or N % S:
        raise ValueError("x's token count must be a whole number of frames")
    code = _dtype_code(x)
    for name, t, shape in (("weight", weight, (2, C)), ("bias", bias, (C,))):
        if t is None:
            continue
        if not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous() or tuple(t.shape) != shape:
            raise ValueError(f"{name} must be a contiguous float32 CUDA tensor {list(shape)}")
    if cache is not None and (not cache.is_cuda or cache.dtype != x.dtype or not cache.is_contiguous()
                              or tuple(cache.shape) != (B, S, C)):
        raise ValueError("cache must be a contiguous CUDA tensor [B, S, C] of x's dtype")
    if out is None:
        out = torch.empty_like(x)
    _check(lib.lcla_temporal_conv(_ptr(x), B, N // S, S, C, _ptr(weight), _ptr(bias), _ptr(cache),
                                  int(bool(save)), _ptr(out), code, _stream(stream, x.device)))
    return out
