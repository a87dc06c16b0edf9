"""The bounded ordering wait of in-place compaction, made to expire on
purpose through the test entry point (include/kvz_testing.h): one chunk
never reports its source rows as read, so the chunk whose rows they are
gives up after 1 ms.  The launch must return, report KVZ_ERR_TIMEOUT (7)
in the device status word, leave every other head exactly compacted, and
leave the context usable.  Nothing here faults, traps or spins unbounded."""
import time

import numpy as np
import pytest
import torch

from kvz_testutil import bits
from oracle import kvz_oracle as orc
from query_agnostic_kv_kvz_b200 import synth

pytestmark = pytest.mark.gpu

kvz = pytest.importorskip("query_agnostic_kv_kvz_b200")

CHUNK = 16          # slots per in-place chunk (the kernel's unit of ordering)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kvz.lib()


def _held_chunk(sel):
    """A chunk k that reads a row some later chunk c > k overwrites (so
    chunk c waits for k), and that c."""
    for k in range(len(sel) // CHUNK):
        later = [int(j) // CHUNK for j in sel[k * CHUNK:(k + 1) * CHUNK] if int(j) // CHUNK > k]
        if later:
            return k, later[0]
    raise AssertionError("no chunk has a later reader")


@pytest.mark.parametrize("d,ratio,hold_head", [(128, 0.3, 2), (64, 0.25, 0)])
def test_in_place_wait_expires_with_timeout_status(d, ratio, hold_head):
    B, n_c = 6, 4096
    g = torch.Generator(device="cuda").manual_seed(d)
    K = torch.randn((B, n_c, d), generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn((B, n_c, d), generator=g, device="cuda").to(torch.bfloat16)
    S = synth.synthetic_scores(B, n_c, seed=d, device="cuda")
    idx, counts, offsets = kvz.kvz_select(S, ratio, "per_head")
    torch.cuda.synchronize()
    ri, rc, ro = orc.select(S.cpu().numpy(), ratio, "per_head")
    np.testing.assert_array_equal(idx.cpu().numpy()[: len(ri)], ri)
    k, c = _held_chunk(ri[ro[hold_head]:ro[hold_head + 1]])
    assert c > k
    Kh, Vh = bits(K), bits(V)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    kvz.kvz_testing_compact_in_place_withhold(K, V, idx, counts, offsets, wait_ns=1_000_000, hold_head=hold_head,
                                              hold_chunk=k, status=status)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert elapsed < 10.0, "the launch did not return promptly (%.1f s)" % elapsed
    assert int(status.item()) == 7, kvz.STATUS.get(int(status.item()))
    Ko, Vo = bits(K), bits(V)
    for b in range(B):
        if b == hold_head:
            continue
        sel = ri[ro[b]:ro[b + 1]]
        np.testing.assert_array_equal(Ko[b, : len(sel)], Kh[b][sel], err_msg="head %d" % b)
        np.testing.assert_array_equal(Vo[b, : len(sel)], Vh[b][sel], err_msg="head %d" % b)
    # the chunks of the held head below the waiting chunk's readers are done
    sel = ri[ro[hold_head]:ro[hold_head + 1]]
    np.testing.assert_array_equal(Ko[hold_head, : k * CHUNK], Kh[hold_head][sel[: k * CHUNK]])

    # the context is still usable: a normal in-place compaction is exact
    K2 = torch.from_numpy(Kh.view(np.int16)).cuda().view(torch.bfloat16)
    V2 = torch.from_numpy(Vh.view(np.int16)).cuda().view(torch.bfloat16)
    status.zero_()
    kvz.kvz_compact(K2, V2, idx, counts, offsets, in_place=True, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    Ko2, Vo2 = bits(K2), bits(V2)
    for b in range(B):
        sel = ri[ro[b]:ro[b + 1]]
        np.testing.assert_array_equal(Ko2[b, : len(sel)], Kh[b][sel])
        np.testing.assert_array_equal(Vo2[b, : len(sel)], Vh[b][sel])


def test_withhold_arguments_are_checked():
    K = torch.zeros((2, 64, 128), dtype=torch.bfloat16, device="cuda")
    V = torch.zeros_like(K)
    idx = torch.zeros(2, dtype=torch.int32, device="cuda")
    counts = torch.ones(2, dtype=torch.int32, device="cuda")
    offsets = torch.tensor([0, 1, 2], dtype=torch.int64, device="cuda")
    for wait_ns, hb, hc in [(10, 0, 0), (2_000_000_000, 0, 0), (1_000_000, 2, 0), (1_000_000, 0, -1)]:
        with pytest.raises(kvz.KvzError) as e:
            kvz.kvz_testing_compact_in_place_withhold(K, V, idx, counts, offsets, wait_ns, hb, hc)
        assert e.value.code == 1
