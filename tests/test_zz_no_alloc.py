"""kvz_score_noalloc: scoring for callers that cannot allocate device memory
(an engine whose memory pool owns the GPU, a plugin without access to the
host program's allocator, a path that must not risk cudaMalloc's implicit
synchronisation).  Its scratch is the library's fixed static device array.

Checked through the C ABI against the regular kvz_score on the same inputs,
within the score tolerance the parity tests use, on two calls in a row (the
second call finds the first call's leftovers in the shared scratch).  This
file is named to be collected last.
"""
import numpy as np
import pytest
import torch

from kvz_testutil import ABS_TOL, REL_FLOOR, REL_TOL

pytestmark = pytest.mark.gpu

kvz = pytest.importorskip("query_agnostic_kv_kvz_b200")
from query_agnostic_kv_kvz_b200 import synth  # noqa: E402

SCRATCH_BYTES = 8 << 20
WORKSPACE = 4


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kvz.lib()


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    err = np.abs(a - b)
    assert err.max() <= ABS_TOL
    big = b > REL_FLOOR
    if big.any():
        assert (err[big] / b[big]).max() <= REL_TOL


@pytest.mark.parametrize("B,G,n_c,n_prompt,d", [
    (8, 4, 8192, 32, 128),     # one chunk: the Llama-3.1-8B-shaped layer
    (64, 4, 8968, 32, 128),    # 64*4*256 rows*4 B = 256 KiB per block -> 32 blocks per chunk, 2 chunks
    (3, 5, 700, 20, 64),
])
def test_noalloc_matches_kvz_score_twice(B, G, n_c, n_prompt, d):
    x = synth.layer_inputs(synth.WORKLOADS["llama8b_layer"], seed=n_c, device="cuda", heads=B, G=G, n_c=n_c,
                           n_prompt=n_prompt, d=d)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = kvz.kvz_score(x["Q"], x["K_ctx"], x["K_in"], status=status)
    first = kvz.kvz_score_noalloc(x["Q"], x["K_ctx"], x["K_in"], status=status)
    second = kvz.kvz_score_noalloc(x["Q"], x["K_ctx"], x["K_in"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _close(first, ref)
    _close(second, ref)
    assert torch.equal(first, second)


def test_noalloc_rejects_heads_beyond_the_scratch():
    # one 256-row block of each (head, group) must fit: B*G*256*4 <= 8 MiB
    B, G, d = 2049, 4, 64                                   # 8196 row groups -> 8.004 MiB
    assert B * G * 256 * 4 > SCRATCH_BYTES
    Q = torch.zeros((B, G, 1, d), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((B, 1, d), dtype=torch.bfloat16, device="cuda")
    S = torch.full((B, 1), -1.0, device="cuda")
    with pytest.raises(kvz.KvzError) as e:
        kvz.kvz_score_noalloc(Q, K, K, S=S)
    assert e.value.code == WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(S == -1.0)                              # nothing was launched
