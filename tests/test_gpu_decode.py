"""GPU parity of decode attention over the pruned cache against the fp64
oracle.  The output is a convex combination of bf16 values computed in fp32:
|d out| <= 1e-4 + 1e-4 |out| and |d lse2| <= 1e-4."""
import numpy as np
import pytest
import torch

from kvz_testutil import f64
from oracle import kvz_oracle as orc
from query_agnostic_kv_kvz_b200 import synth

pytestmark = pytest.mark.gpu

kvz = pytest.importorskip("query_agnostic_kv_kvz_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kvz.lib()


def _cache(B, n_c, d, ratio, mode, seed, skew=False):
    g = torch.Generator(device="cuda").manual_seed(seed)
    K = (torch.randn((B, n_c, d), generator=g, device="cuda") * 1.5).to(torch.bfloat16)
    V = torch.randn((B, n_c, d), generator=g, device="cuda").to(torch.bfloat16)
    S = synth.synthetic_scores(B, n_c, seed=seed, device="cuda")
    if skew:                                   # global mode: head 1 keeps nothing, head 0 a lot
        S[1] = 0.0
        S[0] *= 10.0
    idx, counts, offsets = kvz.kvz_select(S, ratio, mode)
    rows = max(1, int(offsets[-1].item()))
    Ko, Vo = kvz.kvz_compact(K, V, idx, counts, offsets, out_rows=rows)
    return Ko, Vo, counts, offsets


def _check(q, Ko, Vo, counts, offsets, n_c, scale):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse2 = kvz.kvz_decode(q, Ko, Vo, counts, offsets, n_c, scale=scale, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ro, rl = orc.decode_attention(f64(q), f64(Ko), f64(Vo), counts.cpu().numpy(), offsets.cpu().numpy(), scale)
    o = out.cpu().double().numpy()
    assert np.all(np.abs(o - ro) <= 1e-4 + 1e-4 * np.abs(ro)), np.abs(o - ro).max()
    lg = lse2.cpu().double().numpy()
    fin = np.isfinite(rl)
    assert np.array_equal(np.isneginf(lg), ~fin)
    assert np.all(np.abs(lg[fin] - rl[fin]) <= 1e-4)
    return o


@pytest.mark.parametrize("B,G,n_c,d,ratio,mode", [
    (1, 4, 100, 128, 0.3, "per_head"),      # 30 keys: one partial tile
    (8, 4, 8192, 128, 0.3, "per_head"),     # the Llama-3.1-8B layer's pruned cache (2457 keys per head)
    (3, 8, 5000, 64, 0.2, "global"),
    (5, 5, 777, 128, 1.0, "per_head"),      # nothing evicted
    (2, 1, 3, 128, 0.34, "per_head"),       # one key per head
    (64, 5, 32768, 128, 0.25, "per_head"),  # many heads, many splits
])
def test_decode_matches_oracle(B, G, n_c, d, ratio, mode):
    Ko, Vo, counts, offsets = _cache(B, n_c, d, ratio, mode, seed=B * 13 + n_c)
    q = torch.randn((B, G, d), generator=torch.Generator(device="cuda").manual_seed(n_c), device="cuda")
    q = q.to(torch.bfloat16)
    _check(q, Ko, Vo, counts, offsets, n_c, 1.0 / np.sqrt(d))


def test_decode_empty_head_gives_zero():
    B, G, n_c, d = 3, 4, 2000, 128
    Ko, Vo, counts, offsets = _cache(B, n_c, d, 0.1, "global", seed=5, skew=True)
    assert int(counts[1].item()) == 0
    q = torch.randn((B, G, d), device="cuda").to(torch.bfloat16)
    o = _check(q, Ko, Vo, counts, offsets, n_c, 0.088)
    assert np.all(o[1] == 0)


def test_decode_on_full_cache_equals_attention_over_all_keys():
    # counts = n_c and offsets = b*n_c make the original [B, n_c, d] cache a
    # packed one: the decode is plain attention over every key
    B, G, n_c, d = 2, 4, 3000, 128
    g = torch.Generator(device="cuda").manual_seed(9)
    K = torch.randn((B, n_c, d), generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn((B, n_c, d), generator=g, device="cuda").to(torch.bfloat16)
    counts = torch.full((B,), n_c, dtype=torch.int32, device="cuda")
    offsets = torch.arange(B + 1, dtype=torch.int64, device="cuda") * n_c
    q = torch.randn((B, G, d), generator=g, device="cuda").to(torch.bfloat16)
    _check(q, K.view(B * n_c, d), V.view(B * n_c, d), counts, offsets, n_c, 0.09)


def test_decode_reports_count_above_bound():
    B, G, n_c, d = 2, 4, 500, 128
    Ko, Vo, counts, offsets = _cache(B, n_c, d, 0.5, "per_head", seed=3)
    q = torch.randn((B, G, d), device="cuda").to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvz.kvz_decode(q, Ko, Vo, counts, offsets, 100, status=status)     # counts are 250 > 100
    torch.cuda.synchronize()
    assert int(status.item()) == 1


def _packed(counts_list, d, seed):
    """A packed cache with the given per-head counts (rows of head b follow those of head b-1)."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    rows = max(1, sum(counts_list))
    Ko = (torch.randn((rows, d), generator=g, device="cuda") * 1.5).to(torch.bfloat16)
    Vo = torch.randn((rows, d), generator=g, device="cuda").to(torch.bfloat16)
    counts = torch.tensor(counts_list, dtype=torch.int32, device="cuda")
    offsets = torch.zeros(len(counts_list) + 1, dtype=torch.int64, device="cuda")
    offsets[1:] = torch.cumsum(counts.long(), 0)
    return Ko, Vo, counts, offsets


@pytest.mark.parametrize("counts_list,n_c,G", [
    ([131072] + [37] * 7, 131072, 8),             # one head holds nearly all rows: its splits reach the cap
    ([0, 20000, 0, 64, 65, 1, 0, 3000], 20000, 4),  # empty heads between uneven ones, tile-edge counts
    ([n % 300 for n in range(1000)], 300, 2),     # more heads than CTAs in two waves
])
def test_decode_uneven_heads(counts_list, n_c, G):
    d = 128
    Ko, Vo, counts, offsets = _packed(counts_list, d, seed=len(counts_list))
    B = len(counts_list)
    q = torch.randn((B, G, d), generator=torch.Generator(device="cuda").manual_seed(B), device="cuda")
    o = _check(q.to(torch.bfloat16), Ko, Vo, counts, offsets, n_c, 0.088)
    for b, c in enumerate(counts_list):
        if c == 0:
            assert np.all(o[b] == 0)
