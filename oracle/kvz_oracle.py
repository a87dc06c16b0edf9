"""Plain, slow CPU oracle of the KVzip hot path.  TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import this module.  The product path (the CUDA library and
its Python binding) never calls it and shares no code with it.

What it computes (KVzip analysis report, §3.2 "KV importance scoring"):
for one KV head with grouped queries Q (G x n_in x d) of the repeat-prompt +
context input and keys K = [K_ctx ; K_in] ((n_c + n_in) x d),

    A = Softmax(scale * Q K^T)        per query row, over the visible keys
    S[j] = max_{g, i} A[g, i, j]      for the n_c context keys j

The pages write Softmax(Q K^T) with no scale and no mask.  Readings taken here
(each listed with its reason in the design notes):
  * the logits are multiplied by ``scale`` (the usual 1/sqrt(d));
  * the reconstruction forward pass is a causal LM pass: input position i
    (0-based, repeat prompt first, then the context) sees all n_c context keys
    and the input keys 0..i, its own position included;
  * each row is normalised over every key it sees (context and input), and
    only then sliced to the context columns (§3.2 slices A, not the logits);
  * every input row, repeat-prompt rows included, enters the max.

Selection (§4.1 "eviction structure": keep the r% highest scores across all
heads; SelKV page §3.1 sets the kept count to floor(rho * n)) and compaction
(§2.1: the pruned cache is a subset of the full cache) are written as a stable
sort and a fancy-index gather.

Arithmetic is float64 throughout.  Inputs that are bf16 on the device are
decoded exactly from their bit patterns (``bf16_bits_to_f64``).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "bf16_bits_to_f64",
    "row_logits",
    "row_lse",
    "score",
    "chunk_bounds",
    "score_chunked",
    "keep_count",
    "select",
    "head_scores",
    "select_heads",
    "decode_attention",
    "select_protected",
    "quantize_rows",
    "compact_quantized",
    "compact",
    "visible_pairs",
]


# ---------------------------------------------------------------------------
# Input decoding
# ---------------------------------------------------------------------------
def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact float64 value of bfloat16 bit patterns (uint16 / int16 array).

    A bfloat16 is the upper half of an IEEE binary32, so shifting the 16 bits
    into the high half of a 32-bit word gives the same number as a float32.
    """
    b = np.asarray(bits)
    if b.dtype not in (np.uint16, np.int16):
        raise TypeError("expected uint16/int16 bit patterns, got %s" % b.dtype)
    u32 = b.view(np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Scoring (KVzip §3.2)
# ---------------------------------------------------------------------------
def _check_head(Q, K_ctx, K_in):
    Q = np.asarray(Q, dtype=np.float64)
    K_ctx = np.asarray(K_ctx, dtype=np.float64)
    K_in = np.asarray(K_in, dtype=np.float64)
    if Q.ndim != 3 or K_ctx.ndim != 2 or K_in.ndim != 2:
        raise ValueError("expected Q[G,n_in,d], K_ctx[n_c,d], K_in[n_in,d]")
    G, n_in, d = Q.shape
    if K_in.shape != (n_in, d) or K_ctx.shape[1] != d:
        raise ValueError("shape mismatch between Q, K_ctx and K_in")
    return Q, K_ctx, K_in


def row_logits(q, K_ctx, K_in, i, scale):
    """Logits z_u = scale * <q, k_u> of input row i over the keys it sees.

    The unified key index u runs over the n_c context keys, then the input
    keys; input row i sees u < n_c + i + 1 (causal, own position included).
    Returns a float64 vector of length n_c + i + 1.
    """
    q = np.asarray(q, dtype=np.float64)
    K_ctx = np.asarray(K_ctx, dtype=np.float64)
    K_in = np.asarray(K_in, dtype=np.float64)
    keys = np.concatenate([K_ctx, K_in[: i + 1]], axis=0)
    return float(scale) * (keys @ q)


def row_lse(q, K_ctx, K_in, i, scale):
    """Natural log-sum-exp of row i's visible logits (stable: max + log sum)."""
    z = row_logits(q, K_ctx, K_in, i, scale)
    m = np.max(z)
    return float(m + np.log(np.sum(np.exp(z - m))))


def score(Q, K_ctx, K_in, scale, rows=None, row_block=256):
    """S[j] = max over (g, i) of softmax-row value A[g, i, j], j < n_c.

    Q: [G, n_in, d]; K_ctx: [n_c, d]; K_in: [n_in, d]; scale: the logit
    multiplier (a float32 value on the device; promoted here, not recomputed).
    ``rows`` = (i_begin, i_end) restricts the max to input rows in that range
    (each row is still normalised over all keys it sees); None = all rows.
    Rows are visited ``row_block`` at a time only to bound memory: every row's
    softmax is computed whole, and the max over rows is exact in any order.
    """
    Q, K_ctx, K_in = _check_head(Q, K_ctx, K_in)
    G, n_in, d = Q.shape
    n_c = K_ctx.shape[0]
    scale = float(scale)
    i_begin, i_end = (0, n_in) if rows is None else (int(rows[0]), int(rows[1]))
    K_all = np.concatenate([K_ctx, K_in], axis=0)  # unified key index u
    u = np.arange(n_c + n_in)
    S = np.zeros(n_c, dtype=np.float64)
    for r0 in range(i_begin, i_end, row_block):
        r1 = min(i_end, r0 + row_block)
        i = np.arange(r0, r1)
        Z = scale * (Q[:, r0:r1, :] @ K_all.T)                 # [G, rows, keys]
        visible = u[None, :] <= (n_c + i)[:, None]          # [rows, keys]
        Z = np.where(visible[None, :, :], Z, -np.inf)
        m = np.max(Z, axis=2, keepdims=True)                 # finite: n_c >= 1
        lse = m + np.log(np.sum(np.exp(Z - m), axis=2, keepdims=True))
        A_ctx = np.exp(Z[:, :, :n_c] - lse)                  # slice after softmax
        S = np.maximum(S, A_ctx.max(axis=(0, 1)))
    return S


# ---------------------------------------------------------------------------
# Chunked scoring (KVzip §3.4 "technical challenges": chunk-based scoring)
# ---------------------------------------------------------------------------
def chunk_bounds(n_c, m):
    """Context positions [c0, c1) of each chunk: fixed length m, the last one
    shorter when m does not divide n_c."""
    n_c, m = int(n_c), int(m)
    if n_c < 1 or m < 1:
        raise ValueError("n_c and m must be positive")
    return [(c0, min(n_c, c0 + m)) for c0 in range(0, n_c, m)]


def score_chunked(Q_chunks, K_ctx, K_in_chunks, scale, m):
    """Chunked importance scores S[n_c] (KVzip §3.4).

    The context is cut into chunks of m tokens.  Chunk t (positions [c0, c1),
    m_t = c1 - c0 tokens) is appended to the repeat prompt and reconstructed
    on its own: its input has n_in_t = n_prompt + m_t tokens with grouped
    queries Q_chunks[t] [G, n_in_t, d] and input keys K_in_chunks[t]
    [n_in_t, d], and its attention matrix is n_in_t x (m_t + n_in_t): the
    rows see only the chunk's own m_t cache keys K_ctx[c0:c1] plus the input
    keys (causally, own position included), and each row is normalised over
    exactly those keys.  S on the chunk's positions is the max over (g, i) of
    the rows' values on the chunk's cache keys.
    """
    K_ctx = np.asarray(K_ctx, dtype=np.float64)
    bounds = chunk_bounds(K_ctx.shape[0], m)
    if len(Q_chunks) != len(bounds) or len(K_in_chunks) != len(bounds):
        raise ValueError("one Q and one K_in block per chunk")
    S = np.zeros(K_ctx.shape[0], dtype=np.float64)
    scale = float(scale)
    for (c0, c1), Qt, Kit in zip(bounds, Q_chunks, K_in_chunks):
        Qt = np.asarray(Qt, dtype=np.float64)
        Kit = np.asarray(Kit, dtype=np.float64)
        G, n_in, d = Qt.shape
        if Kit.shape != (n_in, d) or n_in < c1 - c0:
            raise ValueError("chunk inputs must be [G, n_prompt + m_t, d] and [n_prompt + m_t, d]")
        keys = np.concatenate([K_ctx[c0:c1], Kit], axis=0)     # m_t cache keys, then the input keys
        mt = c1 - c0
        for g in range(G):
            for i in range(n_in):
                z = scale * (keys[: mt + i + 1] @ Qt[g, i])
                zmax = np.max(z)
                a = np.exp(z - zmax) / np.sum(np.exp(z - zmax))
                S[c0:c1] = np.maximum(S[c0:c1], a[:mt])
    return S


def visible_pairs(G, n_c, n_in):
    """Number of (query row, key) pairs the causal softmax covers for a head."""
    return G * (n_in * n_c + n_in * (n_in + 1) // 2)


# ---------------------------------------------------------------------------
# Selection (KVzip §4.1; keep count floor(rho*n) from the SelKV page §3.1)
# ---------------------------------------------------------------------------
def keep_count(n, ratio):
    """floor(ratio * n) with the product rounded once in IEEE double."""
    ratio = float(ratio)
    if not (0.0 <= ratio <= 1.0):
        raise ValueError("ratio must lie in [0, 1]")
    return int(math.floor(ratio * int(n)))


def select(S, ratio, mode):
    """Top-ratio selection with ties to the lower flattened index.

    S: [B, n_c] float32 scores (>= 0).  mode: "per_head" keeps
    floor(ratio*n_c) of every head; "global" keeps floor(ratio*B*n_c) across
    all heads.  Returns (idx int32 concatenated per head, ascending within a
    head; counts int32 [B]; offsets int64 [B+1]).
    """
    S = np.asarray(S, dtype=np.float32)
    if S.ndim != 2:
        raise ValueError("S must be [B, n_c]")
    B, n_c = S.shape
    if np.isnan(S).any() or (S < 0).any():
        raise ValueError("scores must be non-negative and not NaN")
    if mode == "per_head":
        per_head = []
        k = keep_count(n_c, ratio)
        for b in range(B):
            order = np.argsort(-S[b], kind="stable")  # descending, ties by index
            per_head.append(np.sort(order[:k]))
    elif mode == "global":
        flat = S.reshape(-1)
        k = keep_count(B * n_c, ratio)
        order = np.argsort(-flat, kind="stable")
        kept = np.sort(order[:k])
        heads = kept // n_c
        per_head = [kept[heads == b] - b * n_c for b in range(B)]
    else:
        raise ValueError("mode must be 'per_head' or 'global'")
    counts = np.array([len(x) for x in per_head], dtype=np.int32)
    offsets = np.zeros(B + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    idx = (np.concatenate(per_head) if B else np.zeros(0)).astype(np.int32)
    return idx, counts, offsets


# ---------------------------------------------------------------------------
# Context-independent head scores (KVzip §4.2 "context-independent eviction":
# one static importance per head, the pair scores aggregated by a max along
# the sequence) and head-level eviction
# ---------------------------------------------------------------------------
def head_scores(S):
    """S_head[b] = max over the context positions j of S[b, j]."""
    S = np.asarray(S)
    if S.ndim != 2 or S.shape[1] < 1:
        raise ValueError("S must be [B, n_c] with n_c >= 1")
    return S.max(axis=1)


def select_heads(S_head, ratio, n_c):
    """Head-level eviction: keep the floor(ratio * B) heads with the highest
    head score (ties to the lower head index); a kept head keeps all its n_c
    pairs, an evicted head none.  Returns the selection in the same CSR form
    as ``select`` (idx int32, counts int32 [B], offsets int64 [B+1])."""
    S_head = np.asarray(S_head, dtype=np.float32)
    B = S_head.shape[0]
    order = np.argsort(-S_head, kind="stable")
    kept = np.sort(order[: keep_count(B, ratio)])
    counts = np.zeros(B, dtype=np.int32)
    counts[kept] = int(n_c)
    offsets = np.zeros(B + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    idx = np.tile(np.arange(int(n_c), dtype=np.int32), len(kept))
    return idx, counts, offsets


# ---------------------------------------------------------------------------
# Decode attention over the pruned cache (KVzip §2.1: every later query reads
# the pruned cache K_p, V_p in place of the full one)
# ---------------------------------------------------------------------------
def decode_attention(q, K_out, V_out, counts, offsets, scale):
    """One decode step's attention for each KV head b over its kept rows.

    q: [B, G, d] grouped queries of the new token; K_out, V_out: [rows, d],
    head b's kept keys/values at rows offsets[b] .. offsets[b] + counts[b].
    out[b, g] = sum_j softmax_j(scale * <q[b, g], k_j>) v_j; lse2[b, g] is the
    base-2 log of the softmax denominator (scale folded in).  A head with no
    kept rows gives out = 0 and lse2 = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    K_out = np.asarray(K_out, dtype=np.float64)
    V_out = np.asarray(V_out, dtype=np.float64)
    B, G, d = q.shape
    out = np.zeros((B, G, d))
    lse2 = np.full((B, G), -np.inf)
    for b in range(B):
        r0, n = int(offsets[b]), int(counts[b])
        if n == 0:
            continue
        Kb, Vb = K_out[r0:r0 + n], V_out[r0:r0 + n]
        for g in range(G):
            z = float(scale) * (Kb @ q[b, g])
            zm = np.max(z)
            w = np.exp(z - zm)
            out[b, g] = (w @ Vb) / np.sum(w)
            lse2[b, g] = (zm + np.log(np.sum(w))) / math.log(2.0)
    return out, lse2


# ---------------------------------------------------------------------------
# Protected prefix (KVzip §4.1: the initial system prompt's KV pairs are kept
# intact) and int8 quantisation of the pruned cache (KVzip §4.2, "KV
# quantization": KVzip composes with a quantised cache)
# ---------------------------------------------------------------------------
def select_protected(S, ratio, mode, n_protect):
    """Selection with the first n_protect positions of every head always kept.

    The ratio applies to the other positions: floor(ratio * (n_c - n_protect))
    of them per head, or floor(ratio * B * (n_c - n_protect)) across all heads,
    the highest scores first, ties to the lower flattened index (b, j).
    Returns (idx, counts, offsets) as ``select``."""
    S = np.asarray(S, dtype=np.float32)
    B, n_c = S.shape
    p = int(n_protect)
    if not (0 <= p <= n_c):
        raise ValueError("n_protect must lie in [0, n_c]")
    rest = S[:, p:]
    free = n_c - p
    if mode == "per_head":
        k = keep_count(free, ratio)
        chosen = [np.argsort(-rest[b], kind="stable")[:k] + p for b in range(B)]
    elif mode == "global":
        k = keep_count(B * free, ratio)
        order = np.argsort(-rest.reshape(-1), kind="stable")[:k]
        heads, cols = order // max(free, 1), order % max(free, 1)
        chosen = [cols[heads == b] + p for b in range(B)]
    else:
        raise ValueError("mode must be 'per_head' or 'global'")
    per_head = [np.sort(np.concatenate([np.arange(p), c])).astype(np.int64) for c in chosen]
    counts = np.array([len(x) for x in per_head], dtype=np.int32)
    offsets = np.zeros(B + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    idx = np.concatenate(per_head).astype(np.int32) if B else np.zeros(0, np.int32)
    return idx, counts, offsets


def quantize_rows(X):
    """Symmetric per-row int8 codes of X [rows, d] (float32 arithmetic).

    absmax = max |x| of the row; scale = absmax / 127; code =
    clip(rint(x * (127 / absmax)), -127, 127), rint rounding half to even.
    The divisions and the product are single float32 operations, in this
    order.  A row of zeros gets code 0 and scale 0."""
    X = np.asarray(X, dtype=np.float32)
    absmax = np.max(np.abs(X), axis=1)
    scale = (absmax / np.float32(127.0)).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(absmax > 0, np.float32(127.0) / absmax, np.float32(0.0)).astype(np.float32)
    codes = np.clip(np.rint((X * inv[:, None]).astype(np.float32)), -127, 127).astype(np.int8)
    return codes, scale


def compact_quantized(K_bits, V_bits, idx, counts, offsets):
    """The packed pruned cache as int8 codes with one fp32 scale per row:
    (Kq, K_scale, Vq, V_scale).  K_bits/V_bits are bf16 bit patterns."""
    Kr, Vr = compact(K_bits, V_bits, idx, counts, offsets)
    Kq, Ks = quantize_rows(bf16_bits_to_f64(Kr).astype(np.float32))
    Vq, Vs = quantize_rows(bf16_bits_to_f64(Vr).astype(np.float32))
    return Kq, Ks, Vq, Vs


# ---------------------------------------------------------------------------
# Compaction (KVzip §2.1: the pruned cache is a subset of the full cache)
# ---------------------------------------------------------------------------
def compact(K, V, idx, counts, offsets, out_offsets=None):
    """Gather kept rows in key order.

    K, V: [B, n_c, d] arrays (any dtype; bf16 caches are passed as uint16
    bits so the copy is exact).  Returns (K_out, V_out) as a packed
    [sum(counts), d] pair when out_offsets is None; otherwise arrays sized to
    the largest destination row with each head's rows at out_offsets[b].
    """
    K = np.asarray(K)
    V = np.asarray(V)
    B, n_c, d = K.shape
    counts = np.asarray(counts, dtype=np.int64)
    offsets = np.asarray(offsets, dtype=np.int64)
    dst = offsets if out_offsets is None else np.asarray(out_offsets, dtype=np.int64)
    rows = int(max([dst[b] + counts[b] for b in range(B)] + [0]))
    K_out = np.zeros((rows, d), dtype=K.dtype)
    V_out = np.zeros((rows, d), dtype=V.dtype)
    for b in range(B):
        sel = np.asarray(idx[offsets[b]: offsets[b] + counts[b]], dtype=np.int64)
        K_out[dst[b]: dst[b] + counts[b]] = K[b][sel]
        V_out[dst[b]: dst[b] + counts[b]] = V[b][sel]
    return K_out, V_out
