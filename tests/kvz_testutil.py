"""Helpers shared by the GPU parity tests: bf16 decoding for the oracle, the
score tolerance, and a spawn-based process pool for per-head oracle runs."""
import math
import multiprocessing as mp
import os
import shutil
import tempfile
from concurrent.futures import ProcessPoolExecutor

import numpy as np
import torch

from oracle import kvz_oracle as orc

# Tolerance on S (fixed by the benchmark spec for this hot path): every
# |dS| <= 1e-4 and, where the oracle's S > 1e-3, |dS| / S <= 1e-2.
ABS_TOL = 1e-4
REL_TOL = 1e-2
REL_FLOOR = 1e-3


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 numpy bit patterns (exact)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def f64(t: torch.Tensor) -> np.ndarray:
    return orc.bf16_bits_to_f64(bits(t))


def f32_scale(d: int) -> float:
    """The float32 value of 1/sqrt(d) that the kernels receive."""
    return float(np.float32(1.0 / math.sqrt(d)))


def assert_scores_close(S_gpu, S_ref, what=""):
    S_gpu = np.asarray(S_gpu, dtype=np.float64)
    S_ref = np.asarray(S_ref, dtype=np.float64)
    assert S_gpu.shape == S_ref.shape
    assert np.all(np.isfinite(S_gpu)), what
    err = np.abs(S_gpu - S_ref)
    worst = float(err.max()) if err.size else 0.0
    assert worst <= ABS_TOL, "%s: max |dS| = %.3g at %s" % (what, worst, np.unravel_index(err.argmax(), err.shape))
    big = S_ref > REL_FLOOR
    if big.any():
        rel = float((err[big] / S_ref[big]).max())
        assert rel <= REL_TOL, "%s: max rel dS = %.3g" % (what, rel)


def _score_one(args):
    Qb, Kcb, Kib, scale = args
    return orc.score(orc.bf16_bits_to_f64(Qb), orc.bf16_bits_to_f64(Kcb), orc.bf16_bits_to_f64(Kib), scale)


_POOL = None


def pool():
    """Process pool for oracle heads; spawned, so it is safe after CUDA init."""
    global _POOL
    if _POOL is None:
        n = max(1, min(16, os.cpu_count() or 1))
        _POOL = ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn"))
    return _POOL


def oracle_scores(Q, K_ctx, K_in, scale, heads=None):
    """Oracle S for the given heads of torch bf16 Q[B,G,n_in,d], K_ctx[B,n_c,d], K_in[B,n_in,d]."""
    B = Q.shape[0]
    heads = list(range(B)) if heads is None else list(heads)
    Qb, Kcb, Kib = bits(Q), bits(K_ctx), bits(K_in)
    jobs = [(Qb[b], Kcb[b], Kib[b], scale) for b in heads]
    if len(jobs) == 1 or Q.shape[2] * K_ctx.shape[1] < 4_000_000:
        return np.stack([_score_one(j) for j in jobs])
    return np.stack(list(pool().map(_score_one, jobs)))


# ---------------------------------------------------------------------------
# Whole heads at full size: the oracle's rows split over worker processes.
# Each job is oracle.score(..., rows=(r0, r1)), the max over that row range
# (every row still normalised over all the keys it sees); the ranges' maxima
# merge exactly by np.maximum, which the oracle's own pins cover.
# ---------------------------------------------------------------------------
_HEAD_CACHE = {}


def _rows_job(args):
    qp, kcp, kip, scale, r0, r1, row_block = args
    from threadpoolctl import threadpool_limits
    key = (qp, kcp, kip)
    if key not in _HEAD_CACHE:
        _HEAD_CACHE.clear()
        _HEAD_CACHE[key] = tuple(orc.bf16_bits_to_f64(np.load(p)) for p in key)
    Q, Kc, Ki = _HEAD_CACHE[key]
    with threadpool_limits(1):
        return orc.score(Q, Kc, Ki, scale, rows=(r0, r1), row_block=row_block)


_ROW_POOL = None


def row_pool():
    """Spawned workers for row-split oracle heads: one per core (at most 32),
    fewer if host memory is short (up to 4 GB each at the 128K shapes)."""
    global _ROW_POOL
    if _ROW_POOL is None:
        n = min(32, os.cpu_count() or 1)
        try:
            import psutil
            n = max(1, min(n, int(psutil.virtual_memory().available / (4 << 30))))
        except Exception:
            pass
        _ROW_POOL = ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn"))
    return _ROW_POOL


def oracle_head_rows_parallel(Q_head, Kc_head, Ki_head, scale, rows_per_job=256, row_block=64):
    """Oracle S [n_c] of ONE head from torch bf16 Q [G, n_in, d], K_ctx
    [n_c, d], K_in [n_in, d], its input rows split over row_pool()."""
    tmp = tempfile.mkdtemp(prefix="kvz_oracle_", dir="/dev/shm" if os.path.isdir("/dev/shm") else None)
    try:
        paths = []
        for name, t in (("q", Q_head), ("kc", Kc_head), ("ki", Ki_head)):
            path = os.path.join(tmp, name + ".npy")
            np.save(path, bits(t))
            paths.append(path)
        n_in = Q_head.shape[1]
        jobs = [(*paths, float(scale), r0, min(n_in, r0 + rows_per_job), row_block)
                for r0 in range(0, n_in, rows_per_job)]
        return np.maximum.reduce(list(row_pool().map(_rows_job, jobs)))
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
