"""GPU parity of the sharded global selection's device steps.

The ranks are emulated one after another in this process on one GPU (no
kernel waits on another rank): each "rank" runs kvz_select_dist_begin /
_step / _finish on its own heads, and the exchanges are done here (the
histograms summed on the device, the equal-key totals concatenated).  The
result must be, bit for bit, the slice of kvz_select(KVZ_GLOBAL) over all
heads that falls on each rank, and that selection is the oracle's."""
import numpy as np
import pytest
import torch

from oracle import kvz_oracle as orc
from query_agnostic_kv_kvz_b200 import synth

pytestmark = pytest.mark.gpu

kvz = pytest.importorskip("query_agnostic_kv_kvz_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kvz.lib()


def _sharded(S, splits, ratio):
    B = S.shape[0]
    ranks = []
    for r in range(len(splits) - 1):
        Sr = S[splits[r]:splits[r + 1]].contiguous()
        st = {"S": Sr, "hist": torch.zeros(2048, dtype=torch.int32, device="cuda"),
              "eq": torch.zeros(1, dtype=torch.int64, device="cuda"),
              "ws": torch.empty(kvz.kvz_select_dist_workspace_size(*Sr.shape), dtype=torch.uint8, device="cuda"),
              "status": torch.zeros(1, dtype=torch.int32, device="cuda")}
        kvz.kvz_select_dist_begin(Sr, B, ratio, st["hist"], st["ws"], status=st["status"])
        ranks.append(st)
    for p in range(3):
        total = torch.stack([st["hist"] for st in ranks]).sum(0, dtype=torch.int32)    # the all-reduce
        for st in ranks:
            st["hist"].copy_(total)
            kvz.kvz_select_dist_step(st["S"], p, st["hist"], st["eq"], st["ws"], status=st["status"])
    eq_ranks = torch.cat([st["eq"] for st in ranks])                                 # the all-gather
    out = []
    for r, st in enumerate(ranks):
        b, n_c = st["S"].shape
        k = kvz.kvz_keep_count(B * n_c, ratio)
        idx = torch.empty(max(1, min(k, b * n_c)), dtype=torch.int32, device="cuda")
        cnt = torch.empty(b, dtype=torch.int32, device="cuda")
        off = torch.empty(b + 1, dtype=torch.int64, device="cuda")
        kvz.kvz_select_dist_finish(st["S"], B, ratio, eq_ranks, r, idx, cnt, off, st["ws"], status=st["status"])
        out.append((idx, cnt, off, st))
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("splits,n_c,ratio", [
    ([0, 3, 8], 5000, 0.3),             # two ranks, uneven
    ([0, 1, 4, 9, 16], 20000, 0.1),     # four ranks, chunks of 4096 with a ragged tail
    ([0, 5], 4096 * 3 + 7, 0.25),       # one rank: the steps alone equal one global call
    ([0, 2, 4], 3000, 0.0),             # nothing kept
    ([0, 2, 4], 3000, 1.0),             # everything kept
])
def test_sharded_steps_equal_global_select(splits, n_c, ratio):
    B = splits[-1]
    S = synth.synthetic_scores(B, n_c, seed=B * 31 + n_c, device="cuda")
    S[1, 7:40] = S[2, 100]                                   # a run of exact ties across heads (and ranks)
    ridx, rcnt, roff = kvz.kvz_select(S, ratio, "global")
    torch.cuda.synchronize()
    for r, (idx, cnt, off, st) in enumerate(_sharded(S, splits, ratio)):
        lo, hi = splits[r], splits[r + 1]
        assert int(st["status"].item()) == 0
        assert torch.equal(cnt, rcnt[lo:hi])
        assert torch.equal(off, roff[lo:hi + 1] - roff[lo])
        n = int(off[-1].item())
        assert torch.equal(idx[:n], ridx[int(roff[lo].item()):int(roff[hi].item())])
    # every case, sharded or not, is also the oracle's stable-sort selection
    oidx, ocnt, ooff = orc.select(S.cpu().numpy(), ratio, "global")
    np.testing.assert_array_equal(rcnt.cpu().numpy(), ocnt)
    np.testing.assert_array_equal(roff.cpu().numpy(), ooff)
    np.testing.assert_array_equal(ridx[:int(roff[-1].item())].cpu().numpy(), oidx)
