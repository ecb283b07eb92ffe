"""Host-side helpers for running the routing path data-parallel, one process
per GPU (torch.distributed; NCCL on GPUs, gloo on CPU).

Tokens shard into contiguous ranges; gate, selection, dispatch and combine
need nothing from other ranks.  The one real exchange is the load histogram:
a bias update that must be identical on every rank uses the global counts,
so the per-rank counts are summed with one all-reduce (N int32 values) and
the global assignment total is T_global * K.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def token_range(T: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous, balanced [begin, end) token range of `rank` (sizes differ by at most one)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank / world size")
    base, extra = divmod(T, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def allreduce_counts(counts: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the per-rank expert histograms in place (int32 [N]) and return them."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
    return counts


def global_total(T_local: int, K: int, group=None, device="cpu") -> int:
    """Number of assignments over all ranks (sum of T_local * K)."""
    t = torch.tensor([T_local * K], dtype=torch.int64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return int(t.item())
