"""GPU parity of the protected-prefix selection (KVzip §4.1) and of the int8
compaction (§4.2) against the oracle: both bit-exact (the int8 codes are
decided by the same single float32 operations on both sides)."""
import numpy as np
import pytest
import torch

from kvz_testutil import bits
from oracle import kvz_oracle as orc
from query_agnostic_kv_kvz_b200 import synth

pytestmark = pytest.mark.gpu

kvz = pytest.importorskip("query_agnostic_kv_kvz_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kvz.lib()


@pytest.mark.parametrize("B,n_c,p,ratio,mode", [
    (3, 1000, 16, 0.3, "per_head"), (8, 8192, 64, 0.3, "per_head"), (2, 70000, 500, 0.1, "per_head"),
    (4, 4097, 7, 0.25, "global"), (130, 50000, 100, 0.05, "per_head"), (2, 100, 100, 0.5, "global"),
    (5, 300, 0, 0.4, "global"),
])
def test_select_protected_matches_oracle(B, n_c, p, ratio, mode):
    S = synth.synthetic_scores(B, n_c, seed=B + p, device="cuda")
    S[0, p:p + 10] = float("inf")                  # real +inf scores rank below the protected prefix
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, counts, offsets = kvz.kvz_select_protected(S, ratio, mode, p, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ri, rc, ro = orc.select_protected(S.cpu().numpy(), ratio, mode, p)
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    np.testing.assert_array_equal(offsets.cpu().numpy(), ro)
    np.testing.assert_array_equal(idx.cpu().numpy()[: len(ri)], ri)


@pytest.mark.parametrize("B,n_c,d,ratio,mode", [(3, 1000, 128, 0.3, "per_head"), (4, 4097, 64, 0.25, "global"),
                                                (8, 8192, 128, 0.3, "per_head"), (1, 1, 128, 1.0, "per_head")])
def test_compact_int8_matches_oracle(B, n_c, d, ratio, mode):
    g = torch.Generator(device="cuda").manual_seed(n_c)
    K = (torch.randn((B, n_c, d), generator=g, device="cuda") * torch.rand((B, n_c, 1), generator=g,
                                                                          device="cuda") * 4).to(torch.bfloat16)
    V = torch.randn((B, n_c, d), generator=g, device="cuda").to(torch.bfloat16)
    K[0, 0] = 0.0                                  # a zero row: code 0, scale 0
    S = synth.synthetic_scores(B, n_c, seed=n_c, device="cuda")
    S[0, 0] = float("inf")
    idx, counts, offsets = kvz.kvz_select(S, ratio, mode)
    total = int(offsets[-1].item())
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Kq, Ks, Vq, Vs = kvz.kvz_compact_int8(K, V, idx, counts, offsets, out_rows=max(total, 1), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rKq, rKs, rVq, rVs = orc.compact_quantized(bits(K), bits(V), idx.cpu().numpy(), counts.cpu().numpy(),
                                               offsets.cpu().numpy())
    np.testing.assert_array_equal(Kq[:total].cpu().numpy(), rKq)
    np.testing.assert_array_equal(Vq[:total].cpu().numpy(), rVq)
    np.testing.assert_array_equal(Ks[:total].cpu().numpy().view(np.uint32), rKs.view(np.uint32))
    np.testing.assert_array_equal(Vs[:total].cpu().numpy().view(np.uint32), rVs.view(np.uint32))


def _int8_inputs(B, n_c, d, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    K = (torch.randn((B, n_c, d), generator=g, device="cuda") * torch.rand((B, n_c, 1), generator=g,
                                                                          device="cuda") * 4).to(torch.bfloat16)
    V = torch.randn((B, n_c, d), generator=g, device="cuda").to(torch.bfloat16)
    return K, V


@pytest.mark.parametrize("d", [128, 64])
def test_compact_int8_out_offsets_and_many_units(d):
    # 16 heads x 20000 keys, global keep: uneven heads, many 64-slot units per
    # CTA and a ragged last unit per head; each head's rows land at a padded
    # destination (out_offsets), so the bulk stores start at scattered rows
    B, n_c = 16, 20000
    K, V = _int8_inputs(B, n_c, d, seed=d)
    S = synth.synthetic_scores(B, n_c, seed=d + 1, device="cuda")
    idx, counts, offsets = kvz.kvz_select(S, 0.3, "global")
    cnt = counts.cpu().numpy().astype(np.int64)
    out_off = np.zeros(B, dtype=np.int64)
    out_off[1:] = np.cumsum(cnt[:-1] + 7)          # 7 spare rows after every head
    rows = int(out_off[-1] + cnt[-1] + 7)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Kq = torch.full((rows, d), 99, dtype=torch.int8, device="cuda")
    Vq = torch.full((rows, d), 99, dtype=torch.int8, device="cuda")
    Ks = torch.full((rows,), -1.0, device="cuda")
    Vs = torch.full((rows,), -1.0, device="cuda")
    kvz.kvz_compact_int8(K, V, idx, counts, offsets, out_offsets=torch.from_numpy(out_off).cuda(), Kq=Kq, Vq=Vq,
                         K_scale=Ks, V_scale=Vs, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rKq, rKs, rVq, rVs = orc.compact_quantized(bits(K), bits(V), idx.cpu().numpy(), cnt, offsets.cpu().numpy())
    off = offsets.cpu().numpy()
    hKq, hVq, hKs, hVs = Kq.cpu().numpy(), Vq.cpu().numpy(), Ks.cpu().numpy(), Vs.cpu().numpy()
    for b in range(B):
        o, c, p = int(out_off[b]), int(cnt[b]), int(off[b])
        np.testing.assert_array_equal(hKq[o:o + c], rKq[p:p + c])
        np.testing.assert_array_equal(hVq[o:o + c], rVq[p:p + c])
        np.testing.assert_array_equal(hKs[o:o + c].view(np.uint32), rKs[p:p + c].view(np.uint32))
        np.testing.assert_array_equal(hVs[o:o + c].view(np.uint32), rVs[p:p + c].view(np.uint32))
        assert np.all(hKq[o + c:o + c + 7] == 99) and np.all(hVs[o + c:o + c + 7] == -1.0)   # spare rows untouched


def test_compact_int8_reports_bad_index():
    B, n_c, d = 2, 300, 128
    K, V = _int8_inputs(B, n_c, d, seed=5)
    S = synth.synthetic_scores(B, n_c, seed=6, device="cuda")
    idx, counts, offsets = kvz.kvz_select(S, 0.5, "per_head")
    idx[3] = n_c + 10                              # outside [0, n_c)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvz.kvz_compact_int8(K, V, idx, counts, offsets, out_rows=int(offsets[-1].item()), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1
