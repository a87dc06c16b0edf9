"""Pins of the CPU oracle to facts outside itself (no GPU needed).

Each test checks the oracle against something the KVzip definition or plain
mathematics fixes: hand-worked examples, closed forms, a textbook softmax,
50-digit brute force, invariants of the definition, exhaustive search.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import mpmath
import numpy as np
import pytest
import scipy.special
import torch

from oracle import kvz_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kvzip_hand_examples.json")


def _rand_head(rng, G, n_c, n_in, d, scale_keys=1.0):
    Q = rng.standard_normal((G, n_in, d))
    K_ctx = rng.standard_normal((n_c, d)) * scale_keys
    K_in = rng.standard_normal((n_in, d)) * scale_keys
    return Q, K_ctx, K_in


# --------------------------------------------------------------------------
# Hand-worked examples (tests/golden)
# --------------------------------------------------------------------------
def test_hand_examples():
    with open(GOLDEN) as f:
        data = json.load(f)
    for ex in data["examples"]:
        S = orc.score(np.array(ex["Q"]), np.array(ex["K_ctx"]), np.array(ex["K_in"]),
                      ex["scale"])
        want = np.array([float(Fraction(s)) for s in ex["S"]])
        np.testing.assert_allclose(S, want, rtol=1e-14, atol=0, err_msg=ex["name"])


# --------------------------------------------------------------------------
# Closed forms
# --------------------------------------------------------------------------
@pytest.mark.parametrize("G,n_c,n_in,d", [(1, 1, 1, 4), (4, 7, 12, 8), (3, 33, 40, 16),
                                          (2, 64, 5, 8)])
def test_identical_keys_give_uniform_rows(G, n_c, n_in, d):
    # Every row is uniform over its n_c + i + 1 visible keys; the largest
    # weight a context key gets is at i = 0: S[j] = 1 / (n_c + 1).
    rng = np.random.default_rng(1)
    v = rng.standard_normal(d)
    Q = rng.standard_normal((G, n_in, d)) * 3.0
    S = orc.score(Q, np.tile(v, (n_c, 1)), np.tile(v, (n_in, 1)), 0.37)
    np.testing.assert_allclose(S, 1.0 / (n_c + 1), rtol=1e-13)


def test_zero_queries_give_uniform_rows():
    rng = np.random.default_rng(2)
    n_c, n_in = 19, 23
    _, K_ctx, K_in = _rand_head(rng, 1, n_c, n_in, 8, scale_keys=5.0)
    S = orc.score(np.zeros((3, n_in, 8)), K_ctx, K_in, 1.0)
    np.testing.assert_allclose(S, 1.0 / (n_c + 1), rtol=1e-13)


def test_single_row_equals_textbook_softmax():
    # G = 1, n_in = 1: S is the first n_c entries of one softmax row over the
    # n_c context keys and the single input key.
    rng = np.random.default_rng(3)
    for n_c, d in [(1, 4), (10, 8), (100, 64)]:
        Q, K_ctx, K_in = _rand_head(rng, 1, n_c, 1, d)
        scale = 1.0 / math.sqrt(d)
        z = scale * (np.concatenate([K_ctx, K_in]) @ Q[0, 0])
        np.testing.assert_allclose(orc.score(Q, K_ctx, K_in, scale),
                                   scipy.special.softmax(z)[:n_c], rtol=1e-13)


def test_dominant_key_closed_form():
    # One key aligned with the only query row: S[j*] = 1 / (1 + sum_{u != j*}
    # exp(z_u - z_j*)), tending to 1 as the alignment grows; other keys get
    # S[j] = exp(z_j - z_j*) * S[j*].
    rng = np.random.default_rng(4)
    n_c, d = 12, 8
    Q, K_ctx, K_in = _rand_head(rng, 1, n_c, 1, d)
    for alpha in (1.0, 4.0, 16.0):
        K2 = K_ctx.copy()
        K2[5] = alpha * Q[0, 0]
        z = np.concatenate([K2, K_in]) @ Q[0, 0]
        want5 = 1.0 / (1.0 + sum(math.exp(z[u] - z[5]) for u in range(n_c + 1) if u != 5))
        S = orc.score(Q, K2, K_in, 1.0)
        assert abs(S[5] - want5) <= 1e-14
        for j in range(n_c):
            assert abs(S[j] - math.exp(z[j] - z[5]) * want5) <= 1e-14
    assert S[5] > 1 - 1e-12


# --------------------------------------------------------------------------
# Brute force at 50 digits (independent restatement of the definition)
# --------------------------------------------------------------------------
def _mp_score(Q, K_ctx, K_in, scale):
    mpmath.mp.dps = 50
    G, n_in, d = Q.shape
    n_c = K_ctx.shape[0]
    keys = [list(map(mpmath.mpf, k)) for k in np.concatenate([K_ctx, K_in])]
    best = [mpmath.mpf(0)] * n_c
    sc = mpmath.mpf(scale)
    for g in range(G):
        for i in range(n_in):
            q = list(map(mpmath.mpf, Q[g, i]))
            w = [mpmath.e ** (sc * mpmath.fsum(a * b for a, b in zip(q, keys[u])))
                 for u in range(n_c + i + 1)]
            tot = mpmath.fsum(w)
            for j in range(n_c):
                best[j] = max(best[j], w[j] / tot)
    return np.array([float(x) for x in best])


@pytest.mark.parametrize("seed,G,n_c,n_in,d", [(10, 1, 3, 4, 2), (11, 2, 5, 7, 4),
                                               (12, 3, 16, 8, 8), (13, 4, 9, 2, 3)])
def test_matches_50_digit_brute_force(seed, G, n_c, n_in, d):
    rng = np.random.default_rng(seed)
    Q, K_ctx, K_in = _rand_head(rng, G, n_c, n_in, d, scale_keys=2.0)
    scale = 1.0 / math.sqrt(d)
    np.testing.assert_allclose(orc.score(Q, K_ctx, K_in, scale),
                               _mp_score(Q, K_ctx, K_in, scale), rtol=1e-13, atol=0)


# --------------------------------------------------------------------------
# Invariants of the definition
# --------------------------------------------------------------------------
def test_rows_normalise_and_lse_matches_textbook():
    rng = np.random.default_rng(5)
    G, n_c, n_in, d = 2, 20, 9, 8
    Q, K_ctx, K_in = _rand_head(rng, G, n_c, n_in, d)
    for g in range(G):
        for i in range(n_in):
            z = orc.row_logits(Q[g, i], K_ctx, K_in, i, 0.3)
            assert z.shape == (n_c + i + 1,)
            lse = orc.row_lse(Q[g, i], K_ctx, K_in, i, 0.3)
            assert abs(lse - scipy.special.logsumexp(z)) <= 1e-12
            assert abs(np.exp(z - lse).sum() - 1.0) <= 1e-12


@pytest.mark.parametrize("seed,G,n_c,n_in,d,sc", [(40, 2, 5, 4, 3, 0.7), (41, 1, 9, 6, 8, 1.0 / math.sqrt(8)),
                                                  (42, 3, 1, 3, 2, 1.3)])
def test_row_logits_and_lse_match_brute_force_and_score(seed, G, n_c, n_in, d, sc):
    # The per-row helpers check every lse2 the kernels write, so they are
    # pinned to a 50-digit evaluation of the definition (logits scale*<q,k_u>
    # over the causal key range u < n_c + i + 1, and the log of the softmax
    # denominator) and, through the softmax they define, to score() itself:
    # max over (g, i) of exp(z[:n_c] - lse) must be the oracle's S.
    rng = np.random.default_rng(seed)
    Q, K_ctx, K_in = _rand_head(rng, G, n_c, n_in, d, scale_keys=2.0)
    mpmath.mp.dps = 50
    keys = [list(map(mpmath.mpf, k)) for k in np.concatenate([K_ctx, K_in])]
    msc = mpmath.mpf(sc)
    S_rows = np.zeros(n_c)
    for g in range(G):
        for i in range(n_in):
            q = list(map(mpmath.mpf, Q[g, i]))
            z_mp = [msc * mpmath.fsum(a * b for a, b in zip(q, keys[u])) for u in range(n_c + i + 1)]
            lse_mp = mpmath.log(mpmath.fsum(mpmath.e ** z for z in z_mp))
            z = orc.row_logits(Q[g, i], K_ctx, K_in, i, sc)
            assert z.shape == (n_c + i + 1,)
            np.testing.assert_allclose(z, [float(v) for v in z_mp], rtol=1e-14, atol=1e-15)
            lse = orc.row_lse(Q[g, i], K_ctx, K_in, i, sc)
            assert abs(lse - float(lse_mp)) <= 1e-13 * max(1.0, abs(float(lse_mp)))
            S_rows = np.maximum(S_rows, np.exp(z[:n_c] - lse))
    np.testing.assert_allclose(S_rows, orc.score(Q, K_ctx, K_in, sc), rtol=1e-13, atol=0)


def test_range_permutation_duplication_shift_chunks():
    rng = np.random.default_rng(6)
    G, n_c, n_in, d = 3, 50, 37, 16
    Q, K_ctx, K_in = _rand_head(rng, G, n_c, n_in, d, scale_keys=3.0)
    sc = 0.25
    S = orc.score(Q, K_ctx, K_in, sc)
    assert np.all(S >= 0) and np.all(S <= 1)
    # context keys are visible to every row: permuting them permutes S
    perm = rng.permutation(n_c)
    np.testing.assert_allclose(orc.score(Q, K_ctx[perm], K_in, sc), S[perm], rtol=1e-12)
    # a duplicated query group changes nothing (max over g)
    Q2 = np.concatenate([Q, Q[1:2]], axis=0)
    np.testing.assert_allclose(orc.score(Q2, K_ctx, K_in, sc), S, rtol=1e-13)
    # adding one vector to every key shifts each row's logits by a constant
    v = rng.standard_normal(d)
    np.testing.assert_allclose(orc.score(Q, K_ctx + v, K_in + v, sc), S, rtol=1e-9)
    # the max over rows splits into row chunks exactly
    parts = [orc.score(Q, K_ctx, K_in, sc, rows=(a, min(n_in, a + 16)))
             for a in range(0, n_in, 16)]
    np.testing.assert_array_equal(np.maximum.reduce(parts), S)
    # row_block only bounds memory
    np.testing.assert_allclose(orc.score(Q, K_ctx, K_in, sc, row_block=7), S, rtol=1e-15)


def test_visible_pairs_counts_the_causal_mask():
    G, n_c, n_in = 3, 11, 6
    brute = sum(n_c + i + 1 for g in range(G) for i in range(n_in))
    assert orc.visible_pairs(G, n_c, n_in) == brute


# --------------------------------------------------------------------------
# bf16 decoding
# --------------------------------------------------------------------------
def test_bf16_decoding_exact():
    bits = np.array([0x3F80, 0xC000, 0x7F80, 0x0001, 0x3F81, 0x8000, 0xFF80], np.uint16)
    want = [1.0, -2.0, math.inf, 2.0 ** -133, 1.0 + 2.0 ** -7, -0.0, -math.inf]
    got = orc.bf16_bits_to_f64(bits)
    for a, b in zip(got, want):
        assert a == b and math.copysign(1, a) == math.copysign(1, b)
    rnd = torch.randn(1000).to(torch.bfloat16)
    np.testing.assert_array_equal(orc.bf16_bits_to_f64(rnd.view(torch.int16).numpy()),
                                  rnd.to(torch.float64).numpy())


# --------------------------------------------------------------------------
# Selection
# --------------------------------------------------------------------------
def test_keep_count_is_floor_in_double():
    assert orc.keep_count(256, 0.3) == 76
    assert orc.keep_count(8192, 0.3) == 2457
    assert orc.keep_count(32 * 8 * 32768, 0.3) == 2516582
    assert orc.keep_count(131072, 0.25) == 32768
    assert orc.keep_count(256 * 65537, 0.1) == 1677747
    assert orc.keep_count(10, 0.7) == 7          # 0.7*10 = 7.000000000000001
    assert orc.keep_count(3, 0.1) == 0
    assert orc.keep_count(5, 1.0) == 5 and orc.keep_count(5, 0.0) == 0
    with pytest.raises(ValueError):
        orc.keep_count(5, 1.5)


def _canonical_by_exchange(vals, k):
    """The unique k-subset in which every kept entry beats every dropped one
    (greater value, or equal value and lower index), found by exhaustion."""
    n = len(vals)
    found = []
    for sub in itertools.combinations(range(n), k):
        kept = set(sub)
        ok = all((vals[a] > vals[b]) or (vals[a] == vals[b] and a < b)
                 for a in kept for b in range(n) if b not in kept)
        if ok:
            found.append(sub)
    assert len(found) == 1
    return list(found[0])


def test_select_matches_exhaustive_search():
    rng = np.random.default_rng(7)
    for trial in range(30):
        B, n_c = int(rng.integers(1, 4)), int(rng.integers(1, 7))
        S = rng.choice(np.array([0.0, 0.25, 0.5, 1.0, np.inf], np.float32), size=(B, n_c))
        ratio = float(rng.choice([0.0, 0.2, 0.3, 0.5, 0.75, 1.0]))
        for mode in ("per_head", "global"):
            idx, counts, offsets = orc.select(S, ratio, mode)
            if mode == "per_head":
                k = orc.keep_count(n_c, ratio)
                for b in range(B):
                    got = list(idx[offsets[b]:offsets[b + 1]])
                    assert got == _canonical_by_exchange(list(S[b]), k)
            else:
                k = orc.keep_count(B * n_c, ratio)
                want = _canonical_by_exchange(list(S.reshape(-1)), k)
                got = [b * n_c + j for b in range(B) for j in idx[offsets[b]:offsets[b + 1]]]
                assert got == want
            assert offsets[-1] == len(idx) == counts.sum()


def test_select_special_cases():
    S = np.full((3, 10), 0.5, np.float32)
    idx, counts, offsets = orc.select(S, 0.3, "per_head")
    assert list(counts) == [3, 3, 3] and list(idx) == [0, 1, 2] * 3
    idx, counts, offsets = orc.select(S, 0.3, "global")          # first 9 of 30
    assert list(counts) == [9, 0, 0] and list(idx) == list(range(9))
    idx, counts, _ = orc.select(S, 0.0, "global")
    assert len(idx) == 0 and list(counts) == [0, 0, 0]
    idx, counts, _ = orc.select(S, 1.0, "per_head")
    assert list(idx) == list(range(10)) * 3
    S2 = np.array([[0.1, -0.0, 0.0, np.inf]], np.float32)       # -0 ties with +0
    idx, _, _ = orc.select(S2, 0.75, "per_head")
    assert list(idx) == [0, 1, 3]
    with pytest.raises(ValueError):
        orc.select(np.array([[np.nan, 1.0]], np.float32), 0.5, "global")


# --------------------------------------------------------------------------
# Compaction
# --------------------------------------------------------------------------
def test_compact_gathers_in_order():
    rng = np.random.default_rng(8)
    B, n_c, d = 3, 9, 4
    K = rng.integers(0, 2 ** 16, (B, n_c, d)).astype(np.uint16)
    V = rng.integers(0, 2 ** 16, (B, n_c, d)).astype(np.uint16)
    idx, counts, offsets = orc.select(rng.random((B, n_c)).astype(np.float32), 1.0, "per_head")
    K_out, V_out = orc.compact(K, V, idx, counts, offsets)
    np.testing.assert_array_equal(K_out, K.reshape(-1, d))      # identity at ratio 1
    np.testing.assert_array_equal(V_out, V.reshape(-1, d))
    S = rng.random((B, n_c)).astype(np.float32)
    idx, counts, offsets = orc.select(S, 0.4, "global")
    K_out, V_out = orc.compact(K, V, idx, counts, offsets)
    for b in range(B):
        sel = idx[offsets[b]:offsets[b + 1]]
        assert np.all(np.diff(sel) > 0)
        np.testing.assert_array_equal(K_out[offsets[b]:offsets[b + 1]], K[b][sel])
        np.testing.assert_array_equal(V_out[offsets[b]:offsets[b + 1]], V[b][sel])
    out_off = np.array([b * n_c for b in range(B)])
    K2, _ = orc.compact(K, V, idx, counts, offsets, out_offsets=out_off)
    for b in range(B):
        np.testing.assert_array_equal(K2[b * n_c: b * n_c + counts[b]],
                                      K_out[offsets[b]:offsets[b + 1]])


# --------------------------------------------------------------------------
# Chunked scoring (KVzip §3.4): each chunk is reconstructed on its own, its
# rows normalised over the chunk's m_t cache keys plus the visible input keys
# --------------------------------------------------------------------------
def _chunked_inputs(rng, G, n_c, n_prompt, m, d, scale_keys=1.0):
    K_ctx = rng.standard_normal((n_c, d)) * scale_keys
    Qs, Kis = [], []
    for c0, c1 in orc.chunk_bounds(n_c, m):
        n_in = n_prompt + (c1 - c0)
        Qs.append(rng.standard_normal((G, n_in, d)))
        Kis.append(rng.standard_normal((n_in, d)) * scale_keys)
    return Qs, K_ctx, Kis


def test_chunk_bounds():
    assert orc.chunk_bounds(7, 3) == [(0, 3), (3, 6), (6, 7)]
    assert orc.chunk_bounds(6, 3) == [(0, 3), (3, 6)]
    assert orc.chunk_bounds(5, 8) == [(0, 5)]
    assert orc.chunk_bounds(170000, 2048)[-1] == (169984, 170000)     # 83 full chunks and a 16-token tail


@pytest.mark.parametrize("G,n_c,n_prompt,m,d", [(2, 10, 3, 4, 8), (1, 9, 0, 3, 4), (3, 20, 5, 7, 16)])
def test_chunked_identical_keys_give_one_over_chunk_plus_one(G, n_c, n_prompt, m, d):
    # every row of chunk t is uniform over its m_t + i + 1 visible keys, so the
    # chunk's cache keys score 1 / (m_t + 1): the normaliser is the chunk's, not n_c
    rng = np.random.default_rng(21)
    v = rng.standard_normal(d)
    Qs, _, Kis = _chunked_inputs(rng, G, n_c, n_prompt, m, d)
    K_ctx = np.tile(v, (n_c, 1))
    Kis = [np.tile(v, (k.shape[0], 1)) for k in Kis]
    S = orc.score_chunked(Qs, K_ctx, Kis, 0.41, m)
    want = np.concatenate([np.full(c1 - c0, 1.0 / (c1 - c0 + 1)) for c0, c1 in orc.chunk_bounds(n_c, m)])
    np.testing.assert_allclose(S, want, rtol=1e-13)


def test_chunked_single_key_chunks_are_two_way_softmaxes():
    # m = 1, no prompt, G = 1: chunk j has one cache key k_j and one input row q_j
    # that sees k_j and its own input key: S_j = e^{s k_j.q_j} / (e^{s k_j.q_j} + e^{s kin_j.q_j})
    rng = np.random.default_rng(22)
    n_c, d, s = 6, 5, 0.7
    Qs, K_ctx, Kis = _chunked_inputs(rng, 1, n_c, 0, 1, d)
    S = orc.score_chunked(Qs, K_ctx, Kis, s, 1)
    for j in range(n_c):
        a, b = s * K_ctx[j] @ Qs[j][0, 0], s * Kis[j][0] @ Qs[j][0, 0]
        assert S[j] == pytest.approx(1.0 / (1.0 + math.exp(b - a)), rel=1e-14)


def test_chunked_with_one_chunk_is_the_unchunked_score():
    rng = np.random.default_rng(23)
    G, n_c, n_prompt, d = 3, 17, 4, 8
    Qs, K_ctx, Kis = _chunked_inputs(rng, G, n_c, n_prompt, 64, d)
    assert len(Qs) == 1
    np.testing.assert_allclose(orc.score_chunked(Qs, K_ctx, Kis, 0.3, 64), orc.score(Qs[0], K_ctx, Kis[0], 0.3),
                               rtol=1e-13, atol=0)


def test_chunked_scores_are_local_to_their_chunk():
    rng = np.random.default_rng(24)
    G, n_c, n_prompt, m, d = 2, 11, 3, 4, 8
    Qs, K_ctx, Kis = _chunked_inputs(rng, G, n_c, n_prompt, m, d)
    S0 = orc.score_chunked(Qs, K_ctx, Kis, 0.5, m)
    Qs[1] = Qs[1] * -2.0                     # chunk 1 = positions [4, 8)
    Kis[1] = Kis[1] + 1.0
    S1 = orc.score_chunked(Qs, K_ctx, Kis, 0.5, m)
    assert np.array_equal(S0[:4], S1[:4]) and np.array_equal(S0[8:], S1[8:])
    assert not np.allclose(S0[4:8], S1[4:8])
    assert np.all((S1 >= 0) & (S1 <= 1))


def test_chunked_brute_force_mpmath():
    # n_c = 7 in chunks of 3 (the last holds 1 key), 50-digit evaluation of
    # the per-chunk softmax written out key by key
    rng = np.random.default_rng(25)
    G, n_c, n_prompt, m, d, scale = 2, 7, 2, 3, 4, 0.6
    Qs, K_ctx, Kis = _chunked_inputs(rng, G, n_c, n_prompt, m, d)
    S = orc.score_chunked(Qs, K_ctx, Kis, scale, m)
    mpmath.mp.dps = 50
    sc = mpmath.mpf(scale)
    for (c0, c1), Qt, Kit in zip(orc.chunk_bounds(n_c, m), Qs, Kis):
        keys = [list(map(mpmath.mpf, k)) for k in K_ctx[c0:c1]] + [list(map(mpmath.mpf, k)) for k in Kit]
        mt = c1 - c0
        for j in range(mt):
            best = mpmath.mpf(0)
            for g in range(G):
                for i in range(Qt.shape[1]):
                    q = list(map(mpmath.mpf, Qt[g, i]))
                    w = [mpmath.e ** (sc * mpmath.fsum(a * b for a, b in zip(q, keys[u]))) for u in range(mt + i + 1)]
                    best = max(best, w[j] / mpmath.fsum(w))
            assert abs(S[c0 + j] - float(best)) <= 1e-13 * float(best)


# --------------------------------------------------------------------------
# Head scores and head-level eviction (KVzip §4.2, context-independent)
# --------------------------------------------------------------------------
def test_head_score_is_attained_upper_bound():
    rng = np.random.default_rng(31)
    S = rng.random((6, 50)).astype(np.float32)
    h = orc.head_scores(S)
    for b in range(6):
        assert np.all(S[b] <= h[b]) and h[b] in S[b]     # an upper bound that is attained: the max


def test_head_scores_of_uniform_rows():
    # identical keys: every score is 1/(n_c+1), so is every head score
    rng = np.random.default_rng(32)
    G, n_c, n_in, d = 2, 9, 12, 4
    v = rng.standard_normal(d)
    S = np.stack([orc.score(rng.standard_normal((G, n_in, d)), np.tile(v, (n_c, 1)), np.tile(v, (n_in, 1)), 0.5)
                  for _ in range(3)])
    np.testing.assert_allclose(orc.head_scores(S), 1.0 / (n_c + 1), rtol=1e-13)


@pytest.mark.parametrize("B", [1, 2, 5, 7])
def test_select_heads_exhaustive(B):
    # every kept set of size k over a few score levels: the oracle's set is the
    # one a brute-force search ranks first by (value desc, index asc)
    rng = np.random.default_rng(33 + B)
    n_c = 3
    for trial in range(20):
        S_head = rng.integers(0, 3, B).astype(np.float32) / 2
        for ratio in (0.0, 0.3, 0.5, 1.0):
            k = orc.keep_count(B, ratio)
            # the kept set whose sorted (-score, index) list is lexicographically smallest
            brute = None
            for c in itertools.combinations(range(B), k):
                keyv = sorted([(-float(S_head[i]), i) for i in c])
                if brute is None or keyv < brute[0]:
                    brute = (keyv, c)
            idx, counts, offsets = orc.select_heads(S_head, ratio, n_c)
            kept = [b for b in range(B) if counts[b] == n_c]
            assert tuple(kept) == (brute[1] if brute else ())
            assert set(counts.tolist()) <= {0, n_c} and offsets[-1] == k * n_c
            assert np.array_equal(idx, np.tile(np.arange(n_c), k))


# --------------------------------------------------------------------------
# Decode attention over the pruned cache
# --------------------------------------------------------------------------
def _csr(counts):
    offsets = np.zeros(len(counts) + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    return np.asarray(counts), offsets


def test_decode_single_key_returns_its_value():
    rng = np.random.default_rng(41)
    counts, offsets = _csr([1, 1])
    K, V = rng.standard_normal((2, 8)), rng.standard_normal((2, 8))
    q = rng.standard_normal((2, 3, 8))
    out, lse2 = orc.decode_attention(q, K, V, counts, offsets, 0.7)
    for b in range(2):
        np.testing.assert_allclose(out[b], np.tile(V[b], (3, 1)), rtol=1e-15)
        np.testing.assert_allclose(lse2[b], 0.7 * (q[b] @ K[b]) / math.log(2), rtol=1e-13)


def test_decode_identical_keys_average_the_values():
    rng = np.random.default_rng(42)
    counts, offsets = _csr([5, 0, 3])
    v = rng.standard_normal(6)
    K = np.tile(v, (8, 1))
    V = rng.standard_normal((8, 6))
    q = rng.standard_normal((3, 2, 6)) * 4
    out, lse2 = orc.decode_attention(q, K, V, counts, offsets, 0.3)
    np.testing.assert_allclose(out[0], np.tile(V[:5].mean(axis=0), (2, 1)), rtol=1e-12)
    np.testing.assert_allclose(out[2], np.tile(V[5:].mean(axis=0), (2, 1)), rtol=1e-12)
    assert np.all(out[1] == 0) and np.all(np.isneginf(lse2[1]))        # empty head


def test_decode_on_the_kept_set_is_the_renormalised_full_softmax():
    # attention over a subset equals the full-cache softmax restricted to the
    # subset and renormalised (scipy softmax, an independent routine)
    rng = np.random.default_rng(43)
    n_c, d, G, s = 40, 16, 4, 0.25
    K, V = rng.standard_normal((n_c, d)), rng.standard_normal((n_c, d))
    q = rng.standard_normal((1, G, d))
    keep = np.sort(rng.choice(n_c, 13, replace=False))
    counts, offsets = _csr([len(keep)])
    out, _ = orc.decode_attention(q, K[keep], V[keep], counts, offsets, s)
    for g in range(G):
        p = scipy.special.softmax(s * (K @ q[0, g]))
        pk = p[keep] / p[keep].sum()
        np.testing.assert_allclose(out[0, g], pk @ V[keep], rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------------------
# Protected prefix and int8 rows
# --------------------------------------------------------------------------
def test_int8_rows_golden():
    with open(os.path.join(os.path.dirname(__file__), "golden", "int8_row_quantization.json")) as f:
        g = json.load(f)
    codes, scales = orc.quantize_rows(np.array(g["rows"], dtype=np.float32))
    assert codes.tolist() == g["codes"] and scales.tolist() == g["scales"]


def test_int8_rows_properties():
    rng = np.random.default_rng(51)
    X = (rng.standard_normal((40, 128)) * rng.random((40, 1)) * 5).astype(np.float32)
    X[3] = 0.0
    codes, scales = orc.quantize_rows(X)
    assert codes.dtype == np.int8 and codes[3].tolist() == [0] * 128 and scales[3] == 0
    for r in range(40):
        if r == 3:
            continue
        j = np.argmax(np.abs(X[r]))
        assert abs(int(codes[r, j])) == 127                       # the largest magnitude maps to the end code
        err = np.abs(X[r] - codes[r].astype(np.float64) * scales[r])
        assert np.all(err <= 0.5 * scales[r] * (1 + 1e-5))        # round to nearest: half a step at most
    np.testing.assert_array_equal(orc.quantize_rows(-X)[0], -codes)    # symmetric


@pytest.mark.parametrize("mode", ["per_head", "global"])
def test_select_protected_by_exhaustive_search(mode):
    rng = np.random.default_rng(52 if mode == "per_head" else 53)
    B, n_c, p = 2, 5, 2
    for trial in range(30):
        S = (rng.integers(0, 3, (B, n_c)) / 2).astype(np.float32)
        for ratio in (0.0, 0.34, 0.5, 1.0):
            idx, counts, offsets = orc.select_protected(S, ratio, mode, p)
            kept = {(b, int(j)) for b in range(B) for j in idx[offsets[b]:offsets[b + 1]]}
            assert all((b, j) in kept for b in range(B) for j in range(p))    # the prefix is always there
            free = [(b, j) for b in range(B) for j in range(p, n_c)]
            if mode == "per_head":
                k = orc.keep_count(n_c - p, ratio)
                groups = [[x for x in free if x[0] == b] for b in range(B)]
            else:
                k = orc.keep_count(B * (n_c - p), ratio)
                groups = [free]
            want = set()
            for grp in groups:
                # the k of the group ranked first by (score desc, flattened index asc)
                best = min(itertools.combinations(grp, k), key=lambda c: sorted((-S[x], x) for x in c)) if k else ()
                want |= set(best)
            assert kept - {(b, j) for b in range(B) for j in range(p)} == want


def test_select_protected_zero_prefix_is_select():
    rng = np.random.default_rng(54)
    S = rng.random((3, 40)).astype(np.float32)
    for mode in ("per_head", "global"):
        a = orc.select_protected(S, 0.3, mode, 0)
        b_ = orc.select(S, 0.3, mode)
        for x, y in zip(a, b_):
            np.testing.assert_array_equal(x, y)
