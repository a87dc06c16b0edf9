"""GPU parity of context-independent head scores and head-level eviction
(KVzip §4.2) against the oracle: bit-exact (a max and a selection)."""
import numpy as np
import pytest
import torch

from kvz_testutil import bits, f32_scale
from oracle import kvz_oracle as orc
from query_agnostic_kv_kvz_b200 import synth

pytestmark = pytest.mark.gpu

kvz = pytest.importorskip("query_agnostic_kv_kvz_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kvz.lib()


@pytest.mark.parametrize("B,n_c", [(1, 1), (3, 100), (8, 8192), (5, 9000), (256, 32768), (2, 200001)])
def test_head_score_matches_oracle(B, n_c):
    S = synth.synthetic_scores(B, n_c, seed=B + n_c, device="cuda")
    S[:, :: max(1, n_c // 7)] = 0.0
    if n_c > 10:
        S[0, 3] = -0.0                         # -0 ranks with +0
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    h = kvz.kvz_head_score(S, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert np.array_equal(h.cpu().numpy(), orc.head_scores(np.abs(S.cpu().numpy())))


def test_head_score_reports_invalid():
    S = synth.synthetic_scores(2, 1000, seed=9, device="cuda")
    S[1, 500] = float("nan")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvz.kvz_head_score(S, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 6


@pytest.mark.parametrize("B,n_c,ratio", [(1, 5, 1.0), (8, 100, 0.5), (256, 64, 0.3), (300, 7, 0.0),
                                         (50000, 2, 0.37)])
def test_select_heads_matches_oracle(B, n_c, ratio):
    g = torch.Generator(device="cuda").manual_seed(B)
    S_head = (torch.randint(0, 50, (B,), generator=g, device="cuda").float() / 50)   # many ties
    idx, counts, offsets = kvz.kvz_select_heads(S_head, n_c, ratio)
    ri, rc, ro = orc.select_heads(S_head.cpu().numpy(), ratio, n_c)
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    np.testing.assert_array_equal(offsets.cpu().numpy(), ro)
    np.testing.assert_array_equal(idx.cpu().numpy()[: len(ri)], ri)


def test_head_level_pipeline_compacts_whole_heads():
    """Score a small layer, keep the best half of the heads whole, compact:
    the packed cache is the kept heads' rows in order."""
    w = synth.WORKLOADS["llama8b_layer"]
    x = synth.layer_inputs(w, device="cuda", heads=6, n_c=700, n_prompt=16)
    S = kvz.kvz_score(x["Q"], x["K_ctx"], x["K_in"], scale=f32_scale(w.d))
    h = kvz.kvz_head_score(S)
    idx, counts, offsets = kvz.kvz_select_heads(h, 700, 0.5)
    total = int(offsets[-1].item())
    Ko, Vo = kvz.kvz_compact(x["K_ctx"], x["V"], idx, counts, offsets, out_rows=total)
    torch.cuda.synchronize()
    ri, rc, ro = orc.select_heads(orc.head_scores(S.cpu().numpy()), 0.5, 700)
    rk, rv = orc.compact(bits(x["K_ctx"]), bits(x["V"]), ri, rc, ro)
    np.testing.assert_array_equal(bits(Ko), rk)
    np.testing.assert_array_equal(bits(Vo), rv)
    assert total == 3 * 700
