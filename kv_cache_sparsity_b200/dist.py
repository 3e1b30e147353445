"""Host-side helpers for running one process per GPU.

The decode path shards by sequence and KV head with no exchange step, so the
only cross-rank traffic is timing: every rank measures its own copy of the
work on its own GPU and the slowest rank's time is the job's time.
"""

from __future__ import annotations

import os

import torch


def rank_env():
    """(rank, local_rank, world_size) from the torchrun environment."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, local, world


def dist_on() -> bool:
    return torch.distributed.is_available() and torch.distributed.is_initialized()


def max_over_ranks(x: float, device="cpu") -> float:
    """The largest value of x over all ranks (x itself when not distributed)."""
    if not dist_on():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier():
    if dist_on():
        torch.distributed.barrier()


def shard(n: int, rank: int, world: int) -> range:
    """Contiguous share of n independent items for this rank (sizes differ by <= 1)."""
    lo = n * rank // world
    hi = n * (rank + 1) // world
    return range(lo, hi)
