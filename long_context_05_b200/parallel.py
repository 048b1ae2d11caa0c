"""Multi-GPU plumbing for the DSA path: one process per GPU, no collective on
the data path.

The path is data parallel: prefill query rows only need the shared keys, and
decode sequences are independent problems.  So scaling is by independent
units per rank (weak scaling): every rank runs its own sequences through the
library on its own GPU, and the only collectives are the barrier around the
timed region and the max over ranks of the measured time (torch.distributed,
NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

import torch


def shard_batch(B: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous block of B sequences for `rank`: (first, count).  Ranks
    differ by at most one sequence; every sequence lands on exactly one rank."""
    base, extra = divmod(B, world)
    first = rank * base + min(rank, extra)
    return first, base + (1 if rank < extra else 0)


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s synthetic sequences (independent problems)."""
    return seed + rank


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank measurement (a no-op without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None) -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and torch.device(device).type == "cuda":
            dist.barrier(device_ids=[torch.device(device).index or 0])
        else:
            dist.barrier()
