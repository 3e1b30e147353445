"""Host-side helpers for running one process per GPU.

Every (sequence, KV head) pair is independent through full attention, block
scoring, top-k and reuse attention, so the decode path splits across GPUs
with no exchange step in the data path, in either of two ways:

* by sequence (weak scaling): rank r runs its own batch of sequences of one
  global batch, every KV head of them; the policy of the configured workload
  (rank 0's) is broadcast, so every rank runs the same layers;
* by KV head (strong scaling): rank r holds the KV heads ``shard(Hkv, r,
  world)`` of every sequence of one workload.  The overlap matrix is a ratio
  of two integer sums over index sets (hylra_overlap_counts), so the ranks add
  their counts with one integer all-reduce and every rank derives the same
  matrix, and the same policy, as a single GPU holding every head.

Timing is max-reduced over ranks.
"""

from __future__ import annotations

import os

import numpy as np
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


def sum_over_ranks(*arrays: np.ndarray, device="cpu"):
    """Element-wise integer sums of int64 host arrays over all ranks (the
    arrays themselves when not distributed); exact, in one all-reduce."""
    if not dist_on():
        return tuple(np.asarray(a, dtype=np.int64) for a in arrays)
    flat = np.concatenate([np.asarray(a, dtype=np.int64).ravel() for a in arrays])
    t = torch.from_numpy(flat).to(device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    flat = t.cpu().numpy()
    out, off = [], 0
    for a in arrays:
        n = int(np.asarray(a).size)
        out.append(flat[off:off + n].reshape(np.asarray(a).shape))
        off += n
    return tuple(out)


def pooled_similarity(H, sets: np.ndarray, device="cpu") -> np.ndarray:
    """Overlap matrix of the index sets held by every rank together.

    sets: this rank's profiled index sets, int32 [L, S_rank, k].  Each rank
    counts its own sets with the library (H.overlap_counts), the counts are
    summed over ranks, and the library turns the sums into M: the same matrix,
    bit for bit, as H.similarity over all ranks' sets in one process."""
    inter, total = H.overlap_counts(sets)
    inter, total = sum_over_ranks(inter, total, device=device)
    return H.similarity_from_counts(inter, total)


def broadcast_policy(policy, device="cpu"):
    """Rank 0's policy on every rank (the policy itself when not distributed).
    Every rank calls this once; ranks other than 0 may pass None."""
    if not dist_on():
        return tuple(int(x) for x in policy)
    n = torch.tensor([len(policy) if policy is not None else 0], dtype=torch.int64, device=device)
    torch.distributed.broadcast(n, src=0)
    t = torch.zeros(int(n.item()), dtype=torch.int64, device=device)
    if torch.distributed.get_rank() == 0:
        t.copy_(torch.tensor([int(x) for x in policy], dtype=torch.int64))
    torch.distributed.broadcast(t, src=0)
    return tuple(int(x) for x in t.cpu().tolist())
