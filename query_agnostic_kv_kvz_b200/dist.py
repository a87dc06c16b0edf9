"""Multi-process plumbing for running the hot path on several GPUs.

Every (layer, head) of the KVzip path is independent in per-head mode, so
ranks take disjoint contiguous ranges of heads (or whole replicas of a
workload) and never exchange data; the collectives there are for timing
only (a barrier around the timed region, a max over ranks of the
device-timed durations).

Global mode is the one real exchange (KVzip analysis report, §4.1: the r%
budget spans every head of every layer of a context).  With a context's
heads split over ranks, `select_global_sharded` runs the library's radix
select with the 2048-bin digit histogram summed over ranks three times and
the ranks' threshold-equal counts gathered once, so the kept set is exactly
that of one global selection over all heads.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

__all__ = ["shard_range", "max_over_ranks", "rank_seed", "select_global_sharded", "DeviceSelectSteps"]


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


class DeviceSelectSteps:
    """The steps of the sharded global selection, run by libkvz's kernels
    (kvz_select_dist_begin / _step / _finish) on this rank's GPU."""

    def buffers(self, S_local: torch.Tensor) -> dict:
        import query_agnostic_kv_kvz_b200 as kvz
        dev = S_local.device
        B, n_c = S_local.shape
        return {
            "hist": torch.zeros(2048, dtype=torch.int32, device=dev),      # uint32 bins, summed as int32
            "eq_total": torch.zeros(1, dtype=torch.int64, device=dev),
            "ws": torch.empty(max(1, kvz.kvz_select_dist_workspace_size(B, n_c)), dtype=torch.uint8, device=dev),
        }

    def begin(self, S, B_total, ratio, buf, status):
        import query_agnostic_kv_kvz_b200 as kvz
        kvz.kvz_select_dist_begin(S, B_total, ratio, buf["hist"], buf["ws"], status=status)

    def step(self, S, pass_, buf, status):
        import query_agnostic_kv_kvz_b200 as kvz
        kvz.kvz_select_dist_step(S, pass_, buf["hist"], buf["eq_total"], buf["ws"], status=status)

    def finish(self, S, B_total, ratio, eq_ranks, rank, buf, status):
        import query_agnostic_kv_kvz_b200 as kvz
        B, n_c = S.shape
        k = kvz.kvz_keep_count(B_total * n_c, ratio)
        idx = torch.empty(max(1, min(k, B * n_c)), dtype=torch.int32, device=S.device)
        counts = torch.empty(B, dtype=torch.int32, device=S.device)
        offsets = torch.empty(B + 1, dtype=torch.int64, device=S.device)
        kvz.kvz_select_dist_finish(S, B_total, ratio, eq_ranks, rank, idx, counts, offsets, buf["ws"], status=status)
        return idx, counts, offsets


def select_global_sharded(S_local: torch.Tensor, ratio: float, B_total: Optional[int] = None, group=None,
                          steps=None, status=None):
    """Global top-ratio selection over the heads of one context split across
    the ranks of `group`: rank r holds S_local [B_r, n_c], its heads coming
    after those of ranks 0..r-1.  The result on each rank is the part of
    kvz_select(KVZ_GLOBAL) over all B_total heads that falls on its own heads
    (idx, counts, offsets with offsets from 0).  Every rank must call it.

    Exchanges: three all-reduces (sum) of the 2048-bin histogram, one
    all-gather of one int64 per rank.  B_total, when not given, is the sum of
    the ranks' head counts (one more all-reduce)."""
    grouped = dist.is_available() and dist.is_initialized()
    world = dist.get_world_size(group) if grouped else 1
    rank = dist.get_rank(group) if grouped else 0
    steps = steps if steps is not None else DeviceSelectSteps()
    if B_total is None:
        t = torch.tensor([S_local.shape[0]], dtype=torch.int64, device=S_local.device)
        if world > 1:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
        B_total = int(t.item())
    dev = S_local.device
    empty = S_local.shape[0] == 0          # a rank with no heads still takes part in every exchange
    if empty:
        buf = {"hist": torch.zeros(2048, dtype=torch.int32, device=dev),
               "eq_total": torch.zeros(1, dtype=torch.int64, device=dev)}
    else:
        buf = steps.buffers(S_local)
        steps.begin(S_local, B_total, ratio, buf, status)
    for p in range(3):
        if world > 1:
            dist.all_reduce(buf["hist"], op=dist.ReduceOp.SUM, group=group)
        if empty:
            buf["hist"].zero_()
        else:
            steps.step(S_local, p, buf, status)
    if world > 1:
        parts = [torch.empty_like(buf["eq_total"]) for _ in range(world)]
        dist.all_gather(parts, buf["eq_total"], group=group)
        eq_ranks = torch.cat(parts)
    else:
        eq_ranks = buf["eq_total"].clone()
    if empty:
        return (torch.zeros(0, dtype=torch.int32, device=dev), torch.zeros(0, dtype=torch.int32, device=dev),
                torch.zeros(1, dtype=torch.int64, device=dev))
    return steps.finish(S_local, B_total, ratio, eq_ranks, rank, buf, status)
