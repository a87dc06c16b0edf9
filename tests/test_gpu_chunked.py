"""GPU parity of chunked scoring (KVzip §3.4) against the fp64 oracle.

Each context chunk of m tokens is scored as its own reconstruction: its rows
see the chunk's cache keys plus their own input keys.  Tolerance as for the
plain score: |dS| <= 1e-4 and |dS|/S <= 1e-2 where S > 1e-3.
"""
import numpy as np
import pytest
import torch

from kvz_testutil import assert_scores_close, f32_scale, f64
from oracle import kvz_oracle as orc
from query_agnostic_kv_kvz_b200 import synth

pytestmark = pytest.mark.gpu

kvz = pytest.importorskip("query_agnostic_kv_kvz_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kvz.lib()


def _inputs(B, G, n_c, n_prompt, m, d, seed=0):
    return synth.chunked_inputs(synth.WORKLOADS["llama8b_170k_chunked"], seed=seed, device="cuda", heads=B, G=G,
                                n_c=n_c, n_prompt=n_prompt, d=d, m=m)


def _oracle(x, b, scale, chunks=None):
    """Oracle S of head b on the given chunk indices (all when None); other
    positions are NaN."""
    n_c = x["K_ctx"].shape[1]
    m = x["m"]
    bounds = orc.chunk_bounds(n_c, m)
    T = n_c // m
    Qs, Kis = [], []
    for t in range(len(bounds)):
        if t < T:
            Qs.append(f64(x["Q"][b, t]))
            Kis.append(f64(x["K_in"][b, t]))
        else:
            Qs.append(f64(x["Q_tail"][b]))
            Kis.append(f64(x["K_in_tail"][b]))
    Kc = f64(x["K_ctx"][b])
    if chunks is None:
        return orc.score_chunked(Qs, Kc, Kis, scale, m)
    out = np.full(n_c, np.nan)
    for t in chunks:
        c0, c1 = bounds[t]
        # a chunk's scores depend on its own inputs only: score it as a one-chunk problem
        out[c0:c1] = orc.score_chunked([Qs[t]], Kc[c0:c1], [Kis[t]], scale, c1 - c0)
    return out


def _run(x, status=None):
    return kvz.kvz_score_chunked(x["Q"], x["Q_tail"], x["K_ctx"], x["K_in"], x["K_in_tail"], x["m"],
                                 scale=f32_scale(x["K_ctx"].shape[2]), status=status)


@pytest.mark.parametrize("B,G,n_c,n_prompt,m,d", [
    (2, 4, 700, 16, 256, 128),     # 2 full chunks + a 188-key tail
    (1, 2, 512, 0, 256, 64),       # m divides n_c, no repeat prompt
    (3, 3, 100, 20, 256, 128),     # shorter than one chunk: the tail only
    (2, 4, 1000, 32, 130, 128),    # chunks end 2 keys into a second 128-key tile
    (1, 4, 40, 5, 1, 128),         # one-key chunks
])
def test_chunked_matches_oracle(B, G, n_c, n_prompt, m, d):
    x = _inputs(B, G, n_c, n_prompt, m, d, seed=n_c + m)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    S = _run(x, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    scale = f32_scale(d)
    ref = np.stack([_oracle(x, b, scale) for b in range(B)])
    assert_scores_close(S.cpu().numpy(), ref, "chunked B=%d n_c=%d m=%d" % (B, n_c, m))


def test_one_chunk_equals_the_plain_score():
    # m >= n_c: the single chunk is the whole context, so the result is the
    # plain score's, bit for bit (same kernels, same row order)
    x = _inputs(2, 4, 600, 24, 1000, 128, seed=3)
    S = _run(x)
    Sp = kvz.kvz_score(x["Q_tail"], x["K_ctx"], x["K_in_tail"], scale=f32_scale(128))
    assert torch.equal(S, Sp)


def test_chunked_identical_keys_closed_form():
    B, G, n_c, n_prompt, m, d = 2, 4, 1000, 32, 384, 128
    x = _inputs(B, G, n_c, n_prompt, m, d, seed=4)
    v = x["K_ctx"][:, :1, :]
    x["K_ctx"] = v.expand(B, n_c, d).contiguous()
    x["K_in"] = v[:, None].expand(B, n_c // m, n_prompt + m, d).contiguous()
    x["K_in_tail"] = v.expand(B, n_prompt + n_c % m, d).contiguous()
    S = _run(x).cpu().double().numpy()
    want = np.concatenate([np.full(c1 - c0, 1.0 / (c1 - c0 + 1)) for c0, c1 in orc.chunk_bounds(n_c, m)])
    assert np.abs(S - want[None]).max() <= 1e-4 * want.max()


def test_chunked_170k_workload_sampled_chunks_and_selection():
    """The 170K-key, 2K-chunk workload at full size: three chunks of two heads
    (first, a middle one, the 16-key tail) against the oracle; all scores in
    [0, 1]; selection bit-exact on the GPU's scores."""
    w = synth.WORKLOADS["llama8b_170k_chunked"]
    x = synth.chunked_inputs(w, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    S = _run(x, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    Sh = S.cpu().numpy()
    assert np.all(Sh >= 0) and np.all(Sh <= 1)
    T = w.n_c[0] // w.chunk
    for b in (0, 5):
        ref = _oracle(x, b, f32_scale(w.d), chunks=[0, 41, T])
        sel = ~np.isnan(ref)
        assert_scores_close(Sh[b][sel], ref[sel], "170k chunked head %d" % b)
    idx, counts, offsets = kvz.kvz_select(S, w.ratio, w.mode)
    ri, rc, ro = orc.select(Sh, w.ratio, w.mode)
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    np.testing.assert_array_equal(idx.cpu().numpy()[: len(ri)], ri)
