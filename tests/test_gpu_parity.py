"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded bf16 inputs.

Scores: |dS| <= 1e-4 everywhere and |dS|/S <= 1e-2 where S > 1e-3.
Selection and compaction: bit-exact.  Selection is compared on identical
fp32 scores (the oracle's stable sort run on the scores the GPU selects
from), because a top-k over floating-point scores is discontinuous.
"""
import math

import numpy as np
import pytest
import torch

from kvz_testutil import assert_scores_close, bits, f32_scale, f64, oracle_scores
from oracle import kvz_oracle as orc
from query_agnostic_kv_kvz_b200 import synth

pytestmark = pytest.mark.gpu

kvz = pytest.importorskip("query_agnostic_kv_kvz_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kvz.lib()


def _inputs(B, G, n_c, n_prompt, d, seed=0, name="llama8b_layer"):
    return synth.layer_inputs(synth.WORKLOADS[name], seed=seed, device="cuda", heads=B, G=G, n_c=n_c,
                              n_prompt=n_prompt, d=d)


# ---------------------------------------------------------------------------
# Scoring
# ---------------------------------------------------------------------------
SMALL_SHAPES = [
    # B, G, n_c, n_prompt, d, row_chunk
    (1, 4, 256, 16, 64, 0),        # the tiny reference workload's shape
    (1, 1, 1, 0, 128, 0),          # one context key, one input row
    (2, 3, 127, 5, 128, 0),        # ragged: n_c < tile, n_in not a multiple of 128
    (3, 2, 129, 40, 64, 0),        # ragged: one key past a tile
    (2, 5, 1000, 32, 128, 256),    # G=5 and row chunks of 256 positions
    (1, 1, 300, 0, 128, 0),
    (2, 4, 513, 300, 128, 512),    # chunk larger than a tile, prompt longer than a tile
    (1, 2, 2048, 32, 64, 0),
]


@pytest.mark.parametrize("B,G,n_c,n_prompt,d,row_chunk", SMALL_SHAPES)
def test_score_matches_oracle_small(B, G, n_c, n_prompt, d, row_chunk):
    x = _inputs(B, G, n_c, n_prompt, d, seed=B * 1000 + n_c)
    scale = f32_scale(d)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    S = kvz.kvz_score(x["Q"], x["K_ctx"], x["K_in"], scale=scale, row_chunk=row_chunk, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle_scores(x["Q"], x["K_ctx"], x["K_in"], scale)
    assert_scores_close(S.cpu().numpy(), ref, "score B=%d G=%d n_c=%d" % (B, G, n_c))


@pytest.mark.parametrize("B,G,n_c,n_prompt,d", [(1, 4, 256, 16, 64), (2, 3, 300, 70, 128), (1, 2, 129, 0, 128)])
def test_lse2_matches_oracle_rows(B, G, n_c, n_prompt, d):
    x = _inputs(B, G, n_c, n_prompt, d, seed=7)
    n_in = n_c + n_prompt
    scale = f32_scale(d)
    lse2 = kvz.kvz_score_lse2(x["Q"], x["K_ctx"], x["K_in"], scale=scale).cpu().numpy()
    ld = lse2.shape[-1]
    assert ld == (n_in + 255) // 256 * 256
    Q, Kc, Ki = f64(x["Q"]), f64(x["K_ctx"]), f64(x["K_in"])
    for b in range(B):
        for g in range(G):
            want = np.array([orc.row_lse(Q[b, g, i], Kc[b], Ki[b], i, scale) for i in range(n_in)]) / math.log(2)
            np.testing.assert_allclose(lse2[b, g, :n_in], want, rtol=0, atol=2e-4)
            assert np.all(np.isinf(lse2[b, g, n_in:])) and np.all(lse2[b, g, n_in:] > 0)


def test_row_chunks_merge():
    x = _inputs(2, 4, 777, 600, 128, seed=3)
    S0 = kvz.kvz_score(x["Q"], x["K_ctx"], x["K_in"], row_chunk=0)
    S1 = kvz.kvz_score(x["Q"], x["K_ctx"], x["K_in"], row_chunk=256)
    S2 = kvz.kvz_score(x["Q"], x["K_ctx"], x["K_in"], row_chunk=512)
    # the max over row chunks is exact; a row's lse2 differs between
    # chunkings only in float rounding, when its unit falls in the split
    # last wave of one launch and not of another
    for Sx in (S1, S2):
        a, b = Sx.double().cpu().numpy(), S0.double().cpu().numpy()
        assert np.all(np.abs(a - b) <= 2e-6 * b + 1e-12), np.abs(a - b).max()
    # the same call is bit-identical
    assert torch.equal(S1, kvz.kvz_score(x["Q"], x["K_ctx"], x["K_in"], row_chunk=256))


def test_split_last_wave_matches_whole_units():
    # pass 1 with its partial last wave split over key ranges, and without
    # (no workspace): the same lse2 up to float rounding, and padding +inf
    for (B, G, n_c, n_prompt) in [(3, 5, 4000, 32), (1, 4, 20000, 32), (6, 2, 1500, 300)]:
        x = _inputs(B, G, n_c, n_prompt, 128, seed=n_c)
        n_in = n_c + n_prompt
        i0 = ((n_in // 3) // 256) * 256
        ld = (n_in - i0 + 255) // 256 * 256
        whole = torch.empty((B, G, ld), dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        kvz.lib().kvz_score_lse2(kvz._ptr(x["Q"]), kvz._ptr(x["K_ctx"]), kvz._ptr(x["K_in"]), B, G, n_c, n_in, 128,
                                 float(np.float32(1 / math.sqrt(128))), i0, n_in, kvz._ptr(whole), ld, None, 0,
                                 kvz._ptr(st), kvz._stream(None))
        split = kvz.kvz_score_lse2(x["Q"], x["K_ctx"], x["K_in"], i_begin=i0, scale=float(np.float32(1 / math.sqrt(128))),
                                   status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        a, b = split.cpu().numpy(), whole.cpu().numpy()
        rows = n_in - i0
        np.testing.assert_allclose(a[:, :, :rows], b[:, :, :rows], rtol=0, atol=4e-6 * np.abs(b[:, :, :rows]).max())
        assert np.all(np.isposinf(a[:, :, rows:])) and np.all(np.isposinf(b[:, :, rows:]))


@pytest.mark.parametrize("B,n_c,i0,i1,blocks", [
    # 8 heads x 5 groups x 8 row blocks = 320 units: two full waves of 148
    # CTAs and a split tail; heads 3 and 7 span two waves
    (8, 16384, 4096, 6144, None),
    # one head, 5 groups x 60 row blocks = 300 units: the head spans two
    # full waves (forward, then backward) and a tail split 37 ways (forward)
    (1, 122880, 8192, 23552, [59, 31, 30, 29, 15, 1, 0]),
])
def test_lse2_head_major_waves_match_oracle_rows(B, n_c, i0, i1, blocks):
    # A row pass much shorter than the context runs head-major, and a head
    # whose CTAs span several waves walks its key tiles in alternating
    # directions.  Sampled rows of the (head, group, row block) units against
    # the oracle, with and without the split tail.
    G, n_prompt, d = 5, 32, 128
    x = _inputs(B, G, n_c, n_prompt, d, seed=41 + B)
    n_in = n_c + n_prompt
    scale = f32_scale(d)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ld = i1 - i0
    whole = torch.empty((B, G, ld), dtype=torch.float32, device="cuda")
    kvz.lib().kvz_score_lse2(kvz._ptr(x["Q"]), kvz._ptr(x["K_ctx"]), kvz._ptr(x["K_in"]), B, G, n_c, n_in, d,
                             scale, i0, i1, kvz._ptr(whole), ld, None, 0, kvz._ptr(st), kvz._stream(None))
    split = kvz.kvz_score_lse2(x["Q"], x["K_ctx"], x["K_in"], i_begin=i0, i_end=i1, scale=scale, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    a, w = split.cpu().numpy(), whole.cpu().numpy()
    np.testing.assert_allclose(a[:, :, :ld], w, rtol=0, atol=4e-6 * np.abs(w).max())
    offs = [0, 97, 128, 255]
    for b in range(B):
        Kc, Ki = f64(x["K_ctx"][b]), f64(x["K_in"][b, :i1])
        for g in range(G):
            for blk in (range(ld // 256) if blocks is None else blocks):
                for o in (offs[(b + g + blk) % 2::2] if blocks is None else offs[(g + blk) % 4:][:1]):
                    i = i0 + blk * 256 + o
                    want = orc.row_lse(f64(x["Q"][b, g, i]), Kc, Ki, i, scale) / math.log(2)
                    assert abs(float(a[b, g, i - i0]) - want) <= 2e-4, (b, g, i, float(a[b, g, i - i0]), want)


def test_identical_keys_closed_form():
    # every causal row is uniform over its visible keys: S[j] = 1/(n_c+1)
    B, G, n_c, n_prompt, d = 2, 4, 1000, 32, 128
    x = _inputs(B, G, n_c, n_prompt, d, seed=11)
    v = x["K_ctx"][:, :1, :]
    Kc = v.expand(B, n_c, d).contiguous()
    Ki = v.expand(B, n_c + n_prompt, d).contiguous()
    S = kvz.kvz_score(x["Q"], Kc, Ki).cpu().double().numpy()
    assert np.abs(S - 1.0 / (n_c + 1)).max() <= 1e-4 / (n_c + 1) + 1e-9


@pytest.mark.parametrize("alpha,j", [(6.0, 5000), (12.0, 7950), (25.0, 3000), (12.0, 4110), (40.0, 8000)])
def test_score_extreme_logit_jumps(alpha, j):
    """Pass 1 keeps no per-tile max: a row's reference comes from its first
    tile, and a tile with a logit far above it (terms that overflow, or leave
    the exp2 polynomial's range) is redone against its own max.  Plant a key
    alpha * q_r in a late tile, on an SFU column (j % 16 < 14) or a
    polynomial column (j % 16 >= 14), for logit jumps of roughly 60 to 200
    in log2 units; every score must still match the oracle."""
    B, G, n_c, n_prompt, d = 1, 2, 8192, 40, 128
    x = _inputs(B, G, n_c, n_prompt, d, seed=int(alpha * 100) + j)
    K = x["K_ctx"].clone()
    K[0, j] = (alpha * x["Q"][0, 1, 300].float()).to(torch.bfloat16)
    scale = float(np.float32(1 / math.sqrt(d)))
    S = kvz.kvz_score(x["Q"], K, x["K_in"], scale=scale)
    ref = oracle_scores(x["Q"], K, x["K_in"], scale)
    assert_scores_close(S.cpu().numpy(), ref, "alpha %g key %d" % (alpha, j))
    assert ref[0, j] > 0.99                    # the planted key dominates its row


def test_score_is_deterministic():
    x = _inputs(3, 4, 2000, 32, 128, seed=5)
    S0 = kvz.kvz_score(x["Q"], x["K_ctx"], x["K_in"])
    S1 = kvz.kvz_score(x["Q"], x["K_ctx"], x["K_in"])
    assert torch.equal(S0, S1)


def test_llama8b_layer_full_matches_oracle():
    """The 8-head, 8192-key Llama-3.1-8B-shaped layer, every score checked."""
    w = synth.WORKLOADS["llama8b_layer"]
    x = synth.layer_inputs(w, device="cuda")
    scale = f32_scale(w.d)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    S = kvz.kvz_score(x["Q"], x["K_ctx"], x["K_in"], scale=scale, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle_scores(x["Q"], x["K_ctx"], x["K_in"], scale)
    assert_scores_close(S.cpu().numpy(), ref, "llama8b_layer")


# ---------------------------------------------------------------------------
# Selection (bit-exact on identical fp32 scores)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("B,n_c", [(1, 1), (1, 100), (3, 4097), (8, 8192), (5, 12345), (2, 70000), (130, 50000)])
@pytest.mark.parametrize("ratio", [0.0, 0.1, 0.3, 0.5, 1.0])
@pytest.mark.parametrize("mode", ["per_head", "global"])
def test_select_matches_oracle(B, n_c, ratio, mode):
    S = synth.synthetic_scores(B, n_c, seed=B * 7 + n_c, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, counts, offsets = kvz.kvz_select(S, ratio, mode, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ri, rc, ro = orc.select(S.cpu().numpy(), ratio, mode)
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    np.testing.assert_array_equal(offsets.cpu().numpy(), ro)
    np.testing.assert_array_equal(idx.cpu().numpy()[: len(ri)], ri)


def test_select_all_ties_takes_lowest_indices():
    S = torch.full((4, 5000), 0.25, device="cuda")
    idx, counts, offsets = kvz.kvz_select(S, 0.3, "global")
    k = orc.keep_count(20000, 0.3)
    assert counts.cpu().tolist() == [5000, 1000, 0, 0]
    np.testing.assert_array_equal(idx.cpu().numpy()[:k], np.r_[np.arange(5000), np.arange(1000)])


@pytest.mark.parametrize("n_c,ratio", [(30000, 0.37), (49152, 0.5), (60000, 0.05)])
def test_select_per_head_ties_across_tiles(n_c, ratio):
    """Four score levels: the threshold's ties span several write tiles of
    the one-CTA-per-head path (and the multi-kernel path past its limit)."""
    g = torch.Generator(device="cuda").manual_seed(n_c)
    S = torch.randint(0, 4, (3, n_c), generator=g, device="cuda").float() / 4
    idx, counts, offsets = kvz.kvz_select(S, ratio, "per_head")
    ri, rc, ro = orc.select(S.cpu().numpy(), ratio, "per_head")
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    np.testing.assert_array_equal(offsets.cpu().numpy(), ro)
    np.testing.assert_array_equal(idx.cpu().numpy()[: len(ri)], ri)


def test_select_reports_invalid_scores():
    S = synth.synthetic_scores(2, 1000, seed=1, device="cuda")
    S[1, 17] = float("nan")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvz.kvz_select(S, 0.3, "global", status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 6          # KVZ_ERR_INVALID_SCORE
    S[1, 17] = -1.0
    status.zero_()
    kvz.kvz_select(S, 0.3, "per_head", status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 6


# ---------------------------------------------------------------------------
# Compaction (bit-exact)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("B,n_c,d,ratio,mode", [(1, 1, 128, 1.0, "per_head"), (3, 1000, 128, 0.3, "per_head"),
                                                (4, 4097, 64, 0.25, "global"), (8, 8192, 128, 0.3, "per_head"),
                                                (2, 70000, 128, 0.1, "global"), (5, 333, 64, 0.0, "global")])
def test_compact_out_of_place_matches_oracle(B, n_c, d, ratio, mode):
    g = torch.Generator(device="cuda").manual_seed(n_c)
    K = torch.randn((B, n_c, d), generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn((B, n_c, d), generator=g, device="cuda").to(torch.bfloat16)
    S = synth.synthetic_scores(B, n_c, seed=n_c, device="cuda")
    idx, counts, offsets = kvz.kvz_select(S, ratio, mode)
    total = int(offsets[-1].item())
    K_out, V_out = kvz.kvz_compact(K, V, idx, counts, offsets, out_rows=max(total, 1))
    torch.cuda.synchronize()
    rk, rv = orc.compact(bits(K), bits(V), idx.cpu().numpy(), counts.cpu().numpy(), offsets.cpu().numpy())
    np.testing.assert_array_equal(bits(K_out)[:total], rk)
    np.testing.assert_array_equal(bits(V_out)[:total], rv)


@pytest.mark.parametrize("B,n_c,d,ratio,mode", [(3, 1000, 128, 0.3, "per_head"), (4, 4097, 64, 0.25, "global"),
                                                (2, 70000, 128, 0.9, "global"), (2, 5000, 128, 1.0, "per_head")])
def test_compact_in_place_matches_oracle(B, n_c, d, ratio, mode):
    g = torch.Generator(device="cuda").manual_seed(n_c + 1)
    K = torch.randn((B, n_c, d), generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn((B, n_c, d), generator=g, device="cuda").to(torch.bfloat16)
    S = synth.synthetic_scores(B, n_c, seed=n_c + 1, device="cuda")
    idx, counts, offsets = kvz.kvz_select(S, ratio, mode)
    Kh, Vh = bits(K), bits(V)
    ic, cc, oc = idx.cpu().numpy(), counts.cpu().numpy(), offsets.cpu().numpy()
    # canary: every dropped row becomes a sentinel that must never reach the kept prefix
    for b in range(B):
        keep = np.zeros(n_c, bool)
        keep[ic[oc[b]:oc[b + 1]]] = True
        drop = torch.from_numpy(np.nonzero(~keep)[0]).cuda()
        K.view(torch.int16)[b, drop] = 0x7FC1
        V.view(torch.int16)[b, drop] = 0x7FC1
    Kh, Vh = bits(K), bits(V)
    rk, rv = orc.compact(Kh, Vh, ic, cc, oc)
    K2, V2 = kvz.kvz_compact(K, V, idx, counts, offsets, in_place=True)
    torch.cuda.synchronize()
    assert K2.data_ptr() == K.data_ptr()
    Ko, Vo = bits(K), bits(V)
    for b in range(B):
        c = int(cc[b])
        np.testing.assert_array_equal(Ko[b, :c], rk[oc[b]:oc[b] + c])
        np.testing.assert_array_equal(Vo[b, :c], rv[oc[b]:oc[b] + c])
        np.testing.assert_array_equal(Ko[b, c:], Kh[b, c:])      # rows past the count are untouched
        assert not np.any(Ko[b, :c] == 0x7FC1)


@pytest.mark.parametrize("pattern", ["tail", "head", "blocks", "sparse_tail"])
def test_compact_in_place_structured(pattern):
    """Kept keys clustered so that destination chunks and their source rows
    sit at every distance: all at the end (every row moves far down), all at
    the start (every row stays), alternating blocks of 50, and a thin tail."""
    B, n_c, d = 3, 20000, 128
    j = torch.arange(n_c, device="cuda", dtype=torch.float32)
    if pattern == "tail":
        S, ratio = (j + 1) / n_c, 0.6
    elif pattern == "head":
        S, ratio = (n_c - j) / n_c, 0.6
    elif pattern == "blocks":
        S, ratio = ((j // 50) % 2 == 0).float() + 1e-6 * (n_c - j) / n_c, 0.5
    else:
        S, ratio = (j + 1) / n_c, 0.03
    S = S.expand(B, n_c).contiguous()
    g = torch.Generator(device="cuda").manual_seed(7)
    K = torch.randn((B, n_c, d), generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn((B, n_c, d), generator=g, device="cuda").to(torch.bfloat16)
    idx, counts, offsets = kvz.kvz_select(S, ratio, "per_head")
    Kh, Vh = bits(K), bits(V)
    ic, cc, oc = idx.cpu().numpy(), counts.cpu().numpy(), offsets.cpu().numpy()
    rk, rv = orc.compact(Kh, Vh, ic, cc, oc)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvz.kvz_compact(K, V, idx, counts, offsets, in_place=True, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    Ko, Vo = bits(K), bits(V)
    for b in range(B):
        c = int(cc[b])
        np.testing.assert_array_equal(Ko[b, :c], rk[oc[b]:oc[b] + c])
        np.testing.assert_array_equal(Vo[b, :c], rv[oc[b]:oc[b] + c])
        np.testing.assert_array_equal(Ko[b, c:], Kh[b, c:])


def _pattern_selection(rng, kind, n_c):
    """Ascending kept positions of one head for a selection pattern."""
    if kind == "random":
        keep = rng.random(n_c) < rng.choice([0.02, 0.25, 0.5, 0.9])
    elif kind == "runs":                   # alternating kept / dropped runs of random lengths
        keep, pos, on = np.zeros(n_c, bool), 0, bool(rng.integers(2))
        mean = rng.choice([1.5, 8, 60, 400])
        while pos < n_c:
            L = 1 + int(rng.geometric(1.0 / mean))
            keep[pos:pos + L] = on
            pos, on = pos + L, not on
    elif kind == "tail":
        keep = np.arange(n_c) >= rng.integers(0, n_c)
    elif kind == "head":
        keep = np.arange(n_c) < rng.integers(0, n_c + 1)
    elif kind == "all":
        keep = np.ones(n_c, bool)
    else:                                  # none
        keep = np.zeros(n_c, bool)
    return np.nonzero(keep)[0].astype(np.int32)


@pytest.mark.parametrize("seed", range(16))
def test_compact_in_place_pattern_sweep(seed):
    """In-place compaction over seeded structured selections (its ordering
    wait is what keeps a row from being overwritten before it is read):
    every pattern of every head against the oracle, with every dropped row a
    sentinel that must never reach the kept prefix."""
    rng = np.random.default_rng(1000 + seed)
    B = [1, 3, 7][seed % 3]
    n_c = [17, 1000, 4097, 20000][seed % 4]
    d = [64, 128][(seed // 4) % 2]
    kinds = ["random", "runs", "tail", "head", "all", "none"]
    sels = [_pattern_selection(rng, kinds[(seed + b) % len(kinds)] if b else "runs", n_c) for b in range(B)]
    counts_h = np.array([len(x) for x in sels], np.int32)
    offsets_h = np.zeros(B + 1, np.int64)
    offsets_h[1:] = np.cumsum(counts_h)
    idx_h = np.concatenate(sels).astype(np.int32) if offsets_h[-1] else np.zeros(1, np.int32)
    g = torch.Generator(device="cuda").manual_seed(seed)
    K = torch.randn((B, n_c, d), generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn((B, n_c, d), generator=g, device="cuda").to(torch.bfloat16)
    for b in range(B):
        drop = np.setdiff1d(np.arange(n_c), sels[b])
        if drop.size:
            dt = torch.from_numpy(drop).cuda()
            K.view(torch.int16)[b, dt] = 0x7FC1
            V.view(torch.int16)[b, dt] = 0x7FC1
    Kh, Vh = bits(K), bits(V)
    rk, rv = orc.compact(Kh, Vh, idx_h, counts_h, offsets_h)
    idx, counts, offsets = (torch.from_numpy(idx_h).cuda(), torch.from_numpy(counts_h).cuda(),
                            torch.from_numpy(offsets_h).cuda())
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvz.kvz_compact(K, V, idx, counts, offsets, in_place=True, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    Ko, Vo = bits(K), bits(V)
    for b in range(B):
        c = int(counts_h[b])
        np.testing.assert_array_equal(Ko[b, :c], rk[offsets_h[b]:offsets_h[b] + c])
        np.testing.assert_array_equal(Vo[b, :c], rv[offsets_h[b]:offsets_h[b] + c])
        np.testing.assert_array_equal(Ko[b, c:], Kh[b, c:])
        assert not np.any(Ko[b, :c] == 0x7FC1) and not np.any(Vo[b, :c] == 0x7FC1)


# ---------------------------------------------------------------------------
# The whole path on the two small workloads
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["tiny", "llama8b_layer"])
def test_pipeline_selection_and_compaction_exact(name):
    w = synth.WORKLOADS[name]
    x = synth.layer_inputs(w, device="cuda")
    scale = f32_scale(w.d)
    S = kvz.kvz_score(x["Q"], x["K_ctx"], x["K_in"], scale=scale)
    idx, counts, offsets = kvz.kvz_select(S, w.ratio, w.mode)
    total = int(offsets[-1].item())
    K_out, V_out = kvz.kvz_compact(x["K_ctx"], x["V"], idx, counts, offsets, out_rows=total)
    torch.cuda.synchronize()
    S_np = S.cpu().numpy()
    ri, rc, ro = orc.select(S_np, w.ratio, w.mode)
    np.testing.assert_array_equal(idx.cpu().numpy()[:total], ri)
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    rk, rv = orc.compact(bits(x["K_ctx"]), bits(x["V"]), ri, rc, ro)
    np.testing.assert_array_equal(bits(K_out), rk)
    np.testing.assert_array_equal(bits(V_out), rv)
    if name == "tiny":
        # overlap with the selection made from the oracle's own fp64 scores
        ref_S = oracle_scores(x["Q"], x["K_ctx"], x["K_in"], scale).astype(np.float32)
        oi, _, _ = orc.select(ref_S, w.ratio, w.mode)
        overlap = len(set(oi.tolist()) & set(ri.tolist())) / max(1, len(set(oi.tolist()) | set(ri.tolist())))
        assert overlap > 0.9


# ---------------------------------------------------------------------------
# End to end from host memory
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("B,G,n_c,n_prompt,d,ratio,mode,pinned", [
    (1, 4, 256, 16, 64, 0.3, "per_head", True),
    (11, 2, 700, 32, 128, 0.3, "per_head", True),     # 11 heads in chunks of 2 (the last chunk has 1)
    (11, 2, 700, 32, 128, 0.2, "global", False),      # pageable host memory: correct, serialised
    (3, 4, 2000, 40, 128, 0.0, "per_head", True),     # nothing kept
])
def test_compress_host_matches_device_path(B, G, n_c, n_prompt, d, ratio, mode, pinned):
    x = _inputs(B, G, n_c, n_prompt, d, seed=B * 31 + n_c)
    V = torch.randn((B, n_c, d), generator=torch.Generator(device="cuda").manual_seed(5), device="cuda")
    V = V.to(torch.bfloat16)
    host = {n: (t.cpu().pin_memory() if pinned else t.cpu()) for n, t in
            (("Q", x["Q"]), ("K_ctx", x["K_ctx"]), ("K_in", x["K_in"]), ("V", V))}
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    copy_stream = torch.cuda.Stream()
    out = kvz.kvz_compress_host(host["Q"], host["K_ctx"], host["K_in"], host["V"], ratio, mode, status=status,
                                copy_stream=copy_stream)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # the device path on the same head chunks the host call scores (at most 8
    # chunks of ceil(B / 8) heads), so that S is bit-identical: pass 1's
    # grid, and with it the rounding of its split last wave, follows the
    # heads of a call
    ch = -(-B // min(B, 8))
    S = torch.cat([kvz.kvz_score(x["Q"][h:h + ch], x["K_ctx"][h:h + ch], x["K_in"][h:h + ch])
                   for h in range(0, B, ch)])
    idx, counts, offsets = kvz.kvz_select(S, ratio, mode)
    total = int(offsets[-1].item())
    Ko, Vo = kvz.kvz_compact(x["K_ctx"], V, idx, counts, offsets, out_rows=max(total, 1))
    torch.cuda.synchronize()
    assert torch.equal(out["counts"], counts.cpu()) and torch.equal(out["offsets"], offsets.cpu())
    assert torch.equal(out["idx"][:total], idx.cpu()[:total])
    assert torch.equal(out["K_out"][:total].view(torch.int16), Ko[:total].cpu().view(torch.int16))
    assert torch.equal(out["V_out"][:total].view(torch.int16), Vo[:total].cpu().view(torch.int16))
    # and the selection is the oracle's on these scores
    ri, rc, ro = orc.select(S.cpu().numpy(), ratio, mode)
    np.testing.assert_array_equal(out["idx"].numpy()[:total], ri)
