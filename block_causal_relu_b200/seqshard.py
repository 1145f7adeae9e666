"""Sequence-sharded forward over ranks of a ``torch.distributed`` group.

The sequence is cut into runs of whole blocks, one per rank.  Because every
block reads only the cumulative state of the blocks before it ("Block Causal
Linear Attention", introduction and section "What SANA-Video Actually Uses"),
a rank needs from the ranks before it nothing but the sum of their states:

1. ``shard_begin``: pass A over the rank's tokens and the rank's state total;
2. one all-gather of the totals (B * H * (d+1) * d * 4 bytes per rank);
3. ``shard_end``: the rank's carried-in state (the totals of the ranks before
   it, added in rank order by a kernel), the scan from it and pass C.

The host code here only cuts the sequence and moves the totals; every step of
the arithmetic runs in the library's kernels.
"""
from __future__ import annotations

from typing import List, Optional, Tuple

import torch
import torch.distributed as dist

from . import DEFAULT_EPS, shard_begin, shard_end


def shard_bounds(N: int, block_len: int, world: int) -> List[Tuple[int, int]]:
    """Token ranges [t0, t1) of each rank: the ceil(N / block_len) blocks are
    dealt out in order as evenly as possible (the first ranks take one more
    block when they do not divide), so every range starts on a block boundary
    and only the last non-empty range can end in the ragged last block.
    Ranks beyond the block count get empty ranges."""
    if N < 0 or block_len < 1 or world < 1:
        raise ValueError("need N >= 0, block_len >= 1, world >= 1")
    nb = -(-N // block_len)
    base, extra = divmod(nb, world)
    out, b = [], 0
    for r in range(world):
        nbr = base + (1 if r < extra else 0)
        out.append((min(b * block_len, N), min((b + nbr) * block_len, N)))
        b += nbr
    return out


def gather_totals(total: torch.Tensor, group: Optional[dist.ProcessGroup] = None) -> torch.Tensor:
    """Every rank's total, stacked in rank order: [R, *total.shape].  One
    all-gather over ``group`` (the default group when None); a single process
    without an initialised group is one rank."""
    if not dist.is_available() or not dist.is_initialized():
        return total.unsqueeze(0)
    world = dist.get_world_size(group)
    if world == 1:
        return total.unsqueeze(0)
    out = torch.empty(world * total.numel(), dtype=total.dtype, device=total.device)
    dist.all_gather_into_tensor(out, total.contiguous().view(-1), group=group)
    return out.view(world, *total.shape)


def forward_sharded(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rope_cos: torch.Tensor,
                    rope_sin: torch.Tensor, block_len: int, eps: float = DEFAULT_EPS, *,
                    state_in: Optional[torch.Tensor] = None, group: Optional[dist.ProcessGroup] = None,
                    want_state: bool = True, workspace: Optional[torch.Tensor] = None,
                    out: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """This rank's part of a sequence-sharded forward.

    q, k, v [B, N_r, H, d] hold the rank's tokens, ``shard_bounds(N,
    block_len, world)[rank]`` of the whole sequence, and the tables the rows at
    those absolute positions.  ``state_in`` (same on every rank, or None) is
    the state before the sequence.  Returns (out [B, N_r, H, d], the state
    after the whole sequence, bit-identical on every rank).  All ranks must
    call it together; the work is enqueued on ``stream`` (the current stream
    when None), which the all-gather also follows."""
    rank = dist.get_rank(group) if dist.is_available() and dist.is_initialized() else 0
    ctx = torch.cuda.stream(stream) if stream is not None else torch.cuda.stream(torch.cuda.current_stream(q.device))
    with ctx:
        total, ws = shard_begin(k, v, rope_cos, rope_sin, block_len, workspace=workspace)
        totals = gather_totals(total, group)
        return shard_end(q, k, v, rope_cos, rope_sin, block_len, totals, rank, ws, eps,
                         state_in=state_in, out=out, want_state=want_state)
