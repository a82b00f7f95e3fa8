"""Data-parallel plumbing for the layer (one process per GPU, torch.distributed).

Tokens shard across ranks: rows of X, G, Y and dX are independent, the frozen 4-bit
residual, the stabilizer and the adapter factors are replicated.  The only exchange is
the sum of the adapter gradients dA [r, K] and dB [N, r] (FourTune section 3.2: only
the adapter branch has weight gradients), one all-reduce each per layer.  The tensor
factor g of Q(X) and Q(G) is per rank (each rank quantizes its own shard); dA and dB
use the unquantized X and G, so their sum over shards equals the full-batch gradient.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist


def allreduce_adapter_grads(da: torch.Tensor, db: torch.Tensor, group: Optional[dist.ProcessGroup] = None
                            ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Sum dA and dB over the ranks in place (both ranks take the same two steps)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(da, op=dist.ReduceOp.SUM, group=group)
        dist.all_reduce(db, op=dist.ReduceOp.SUM, group=group)
    return da, db


def max_over_ranks(value: float, device: torch.device, group: Optional[dist.ProcessGroup] = None) -> float:
    """The slowest rank's time (multi-GPU numbers are the max over ranks)."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def token_shard(m_total: int, world: int, rank: int, multiple: int = 128) -> Tuple[int, int]:
    """[start, stop) of this rank's tokens for a fixed global batch (strong scaling);
    shard sizes are multiples of `multiple` (the layer's row tile)."""
    if m_total % multiple:
        raise ValueError("global token count must be a multiple of the row tile")
    tiles = m_total // multiple
    base, extra = divmod(tiles, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start * multiple, stop * multiple
