"""Multi-process plumbing for running the hot path on several GPUs.

Every (layer, head) of the KVzip path is independent in per-head mode, so
ranks take disjoint contiguous ranges of heads (or whole replicas of a
workload) and never exchange data.  The only collectives are for timing:
a barrier around the timed region and a max over ranks of the device-timed
durations.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import torch
import torch.distributed as dist

__all__ = ["shard_range", "max_over_ranks", "rank_seed"]


def shard_range(n: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous [lo, hi) share of n units for `rank` of `world`; sizes
    differ by at most one and earlier ranks take the larger shares."""
    if world < 1 or not (0 <= rank < world) or n < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's independent replica."""
    return seed * 1_000_003 + rank


def max_over_ranks(values: Sequence[float], device=None) -> List[float]:
    """Element-wise max of `values` over all ranks (identity when the
    process group is not initialised)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]
