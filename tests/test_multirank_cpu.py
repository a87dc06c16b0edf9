"""World-size-2 checks of the multi-rank plumbing on CPU (gloo backend)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as tmp

from query_agnostic_kv_kvz_b200.dist import max_over_ranks, rank_seed, shard_range


def test_shard_range_partitions():
    for n in (0, 1, 7, 8, 256, 384):
        for world in (1, 2, 3, 8):
            spans = [shard_range(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            for (a, b), (c, _) in zip(spans, spans[1:]):
                assert b == c
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        lo, hi = shard_range(8 * 32, world, rank)
        times = [1.0 + rank, 10.0 - rank, float(hi - lo)]
        mx = max_over_ranks(times)
        dist.barrier()
        out[rank] = torch.tensor([lo, hi, rank_seed(0, rank)] + mx, dtype=torch.float64)
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_and_reduce():
    world = 2
    port = _free_port()
    out = torch.zeros(world, 6, dtype=torch.float64).share_memory_()
    tmp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    r0, r1 = out[0].tolist(), out[1].tolist()
    assert (r0[0], r0[1], r1[0], r1[1]) == (0, 128, 128, 256)        # disjoint halves
    assert r0[2] != r1[2]                                             # independent seeds
    assert r0[3:] == r1[3:] == [2.0, 10.0, 128.0]                     # max over ranks
