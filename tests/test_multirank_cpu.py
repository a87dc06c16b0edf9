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


# ---------------------------------------------------------------------------
# Sharded global selection: the host orchestration (three histogram
# all-reduces, one all-gather of equal-key totals) driven over gloo with a
# NumPy restatement of the device steps, checked against the oracle's
# global selection over all heads (a stable sort, not a radix select).
# ---------------------------------------------------------------------------
import numpy as np  # noqa: E402

from oracle import kvz_oracle as orc  # noqa: E402
from query_agnostic_kv_kvz_b200.dist import select_global_sharded  # noqa: E402

_SHIFT = (21, 10, 0)
_MASK = (0x7FF, 0x7FF, 0x3FF)


class NumpySelectSteps:
    """The three-digit radix select of the library's step calls, on the
    CPU: digit histograms over keys that match the prefix fixed so far, the
    pick of the digit that holds the k_rem-th largest key, then the keys
    above the threshold T plus the first r_t keys equal to it in flattened
    order, counting those of lower ranks first."""

    def buffers(self, S):
        return {"hist": torch.zeros(2048, dtype=torch.int32), "eq_total": torch.zeros(1, dtype=torch.int64),
                "state": {}}

    @staticmethod
    def _keys(S):
        u = S.numpy().astype(np.float32).view(np.uint32).copy()
        u[u == 0x80000000] = 0
        return u

    def _hist(self, keys, st, p):
        match = (keys & st["mask"]) == st["prefix"]
        d = (keys[match] >> _SHIFT[p]) & _MASK[p]
        return np.bincount(d.astype(np.int64), minlength=2048).astype(np.int32)

    def begin(self, S, B_total, ratio, buf, status):
        keys = self._keys(S).reshape(-1)
        k = orc.keep_count(B_total * S.shape[1], ratio)
        st = buf["state"]
        st.update(prefix=np.uint32(0), mask=np.uint32(0), k_rem=k, keys=keys)
        buf["hist"][:] = torch.from_numpy(self._hist(keys, st, 0) if k > 0 else np.zeros(2048, np.int32))

    def step(self, S, p, buf, status):
        st = buf["state"]
        keys = st["keys"]
        if st["k_rem"] > 0 and not st.get("done"):
            h = buf["hist"].numpy().astype(np.int64)
            nb = 1024 if p == 2 else 2048
            above = 0
            for digit in range(nb - 1, -1, -1):          # highest digit first
                if above + h[digit] >= st["k_rem"]:
                    break
                above += h[digit]
            st["prefix"] = np.uint32(st["prefix"] | (digit << _SHIFT[p]))
            st["mask"] = np.uint32(st["mask"] | (_MASK[p] << _SHIFT[p]))
            st["k_rem"] -= above
        else:
            st["done"] = True
        buf["hist"].zero_()
        if p < 2:
            if not st.get("done"):
                buf["hist"][:] = torch.from_numpy(self._hist(keys, st, p + 1))
        else:
            buf["eq_total"][0] = 0 if st.get("done") else int(np.count_nonzero(keys == st["prefix"]))

    def finish(self, S, B_total, ratio, eq_ranks, rank, buf, status):
        st = buf["state"]
        B, n_c = S.shape
        keys = st["keys"].reshape(B, n_c)
        per_head = []
        if st.get("done"):
            per_head = [np.zeros(0, np.int64) for _ in range(B)]
        else:
            T, r_t = st["prefix"], st["k_rem"]
            e = int(eq_ranks[:rank].sum())
            for b in range(B):
                kept = []
                for j in range(n_c):
                    if keys[b, j] > T:
                        kept.append(j)
                    elif keys[b, j] == T:
                        if e < r_t:
                            kept.append(j)
                        e += 1
                per_head.append(np.array(kept, np.int64))
        counts = np.array([len(x) for x in per_head], np.int32)
        offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
        idx = np.concatenate(per_head).astype(np.int32) if counts.sum() else np.zeros(0, np.int32)
        return torch.from_numpy(idx), torch.from_numpy(counts), torch.from_numpy(offsets)


def _tie_scores(B, n_c, seed):
    """Scores with many exact ties (few distinct values), zeros and +inf."""
    rng = np.random.default_rng(seed)
    S = rng.choice(np.float32([0.0, 0.125, 0.25, 0.5, 1.0, 3.0]), size=(B, n_c)).astype(np.float32)
    S[rng.random((B, n_c)) < 0.3] = rng.random(int((rng.random((B, n_c)) < 0.3).sum()) or 1)[0]
    S[0, :3] = np.inf
    return S


def _sel_worker(rank, world, port, splits, B, n_c, ratio, seed, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        S = torch.from_numpy(_tie_scores(B, n_c, seed))
        lo, hi = splits[rank], splits[rank + 1]
        idx, counts, offsets = select_global_sharded(S[lo:hi].contiguous(), ratio, steps=NumpySelectSteps())
        # this rank's (head, position) pairs, in global head numbering
        pairs = [(lo + b, int(j)) for b in range(hi - lo) for j in idx[offsets[b]:offsets[b + 1]].tolist()]
        out[rank] = pairs
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,splits,ratio", [(2, [0, 3, 8], 0.3), (3, [0, 1, 1, 5], 0.55), (2, [0, 4, 5], 0.0)])
def test_sharded_global_select_matches_oracle(world, splits, ratio):
    B, n_c, seed = splits[-1], 300, world * 7 + len(splits)
    port = _free_port()
    mgr = tmp.Manager()
    out = mgr.dict()
    tmp.spawn(_sel_worker, args=(world, port, splits, B, n_c, ratio, seed, out), nprocs=world, join=True)
    got = sorted(p for r in range(world) for p in out[r])
    ridx, rcounts, roffsets = orc.select(_tie_scores(B, n_c, seed), ratio, "global")
    want = sorted((b, int(j)) for b in range(B) for j in ridx[roffsets[b]:roffsets[b + 1]])
    assert got == want
    assert len(want) == orc.keep_count(B * n_c, ratio)


def test_sharded_global_select_without_a_process_group():
    # one process, no process group: the driver's exchanges reduce to
    # identities and the result is the oracle's global selection
    B, n_c, ratio = 4, 257, 0.4
    S = _tie_scores(B, n_c, seed=11)
    idx, counts, offsets = select_global_sharded(torch.from_numpy(S), ratio, steps=NumpySelectSteps())
    ridx, rcounts, roffsets = orc.select(S, ratio, "global")
    assert counts.tolist() == rcounts.tolist()
    assert offsets.tolist() == roffsets.tolist()
    assert idx.tolist() == ridx.tolist()
