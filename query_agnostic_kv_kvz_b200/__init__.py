"""KVzip query-agnostic KV-cache compression hot path on B200 (sm_100a).

Thin Python binding of the C ABI declared in ``include/kvz.h``: every
function here only checks tensor shapes, allocates outputs/workspace with
torch and calls the same-named C entry point in ``libkvz.so``.  All arithmetic
runs in the library's CUDA kernels; there is no CPU fallback.  If the library
is missing, importing works but every call raises ``KvzLibraryError``.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

__all__ = [
    "KvzError", "KvzLibraryError", "lib", "lib_path", "STATUS", "PER_HEAD", "GLOBAL",
    "kvz_version", "kvz_keep_count", "kvz_score_workspace_size", "kvz_score", "kvz_score_noalloc",
    "kvz_score_lse2", "kvz_score_lse2_workspace_size", "kvz_score_colmax", "kvz_select_workspace_size", "kvz_select",
    "kvz_select_dist_workspace_size", "kvz_select_dist_begin", "kvz_select_dist_step", "kvz_select_dist_finish",
    "kvz_compact_workspace_size", "kvz_compact", "kvz_compress_host_workspace_size", "kvz_compress_host",
    "kvz_score_chunked_workspace_size", "kvz_score_chunked", "kvz_head_score", "kvz_select_heads", "kvz_decode",
    "kvz_select_protected", "kvz_compact_int8", "kvz_testing_compact_in_place_withhold",
]

PER_HEAD = 0
GLOBAL = 1
STATUS = {
    0: "KVZ_OK", 1: "KVZ_ERR_INVALID_ARG", 2: "KVZ_ERR_UNSUPPORTED", 3: "KVZ_ERR_ALIGNMENT",
    4: "KVZ_ERR_WORKSPACE", 5: "KVZ_ERR_CUDA", 6: "KVZ_ERR_INVALID_SCORE", 7: "KVZ_ERR_TIMEOUT",
}

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libkvz.so")


class KvzLibraryError(RuntimeError):
    """libkvz.so is missing or cannot be loaded."""


class KvzError(RuntimeError):
    """A libkvz call returned an error status."""

    def __init__(self, fn: str, code: int):
        super().__init__("%s failed: %s (%d)" % (fn, STATUS.get(code, "?"), code))
        self.code = code


_lib = None

_c = ctypes
_vp, _i64, _i32, _f32, _f64, _sz = _c.c_void_p, _c.c_int64, _c.c_int, _c.c_float, _c.c_double, _c.c_size_t
_SIGS = {
    "kvz_version": (_i32, []),
    "kvz_status_string": (_c.c_char_p, [_i32]),
    "kvz_score_workspace_size": (_sz, [_i64, _i32, _i64, _i64]),
    "kvz_score": (_i32, [_vp, _vp, _vp, _i64, _i32, _i64, _i64, _i32, _f32, _i64, _vp, _vp, _sz, _vp, _vp]),
    "kvz_score_lse2_workspace_size": (_sz, []),
    "kvz_score_lse2": (_i32, [_vp, _vp, _vp, _i64, _i32, _i64, _i64, _i32, _f32, _i64, _i64, _vp, _i64, _vp, _sz,
                              _vp, _vp]),
    "kvz_score_colmax": (_i32, [_vp, _vp, _i64, _i32, _i64, _i64, _i32, _f32, _i64, _i64, _vp, _i64, _vp,
                                _i32, _vp, _vp]),
    "kvz_score_noalloc": (_i32, [_vp, _vp, _vp, _i64, _i32, _i64, _i64, _i32, _f32, _vp, _vp, _vp]),
    "kvz_keep_count": (_i64, [_i64, _f64]),
    "kvz_select_workspace_size": (_sz, [_i64, _i64, _i32]),
    "kvz_select": (_i32, [_vp, _i64, _i64, _f64, _i32, _vp, _i64, _vp, _vp, _vp, _sz, _vp, _vp]),
    "kvz_select_dist_workspace_size": (_sz, [_i64, _i64]),
    "kvz_select_dist_begin": (_i32, [_vp, _i64, _i64, _i64, _f64, _vp, _vp, _sz, _vp, _vp]),
    "kvz_select_dist_step": (_i32, [_vp, _i64, _i64, _i32, _vp, _vp, _vp, _sz, _vp, _vp]),
    "kvz_select_dist_finish": (_i32, [_vp, _i64, _i64, _i64, _f64, _vp, _i32, _vp, _i64, _vp, _vp, _vp, _sz, _vp,
                                      _vp]),
    "kvz_compact_workspace_size": (_sz, [_i64, _i64]),
    "kvz_compact": (_i32, [_vp, _vp, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp]),
    "kvz_select_protected": (_i32, [_vp, _i64, _i64, _f64, _i32, _i64, _vp, _i64, _vp, _vp, _vp, _sz, _vp, _vp]),
    "kvz_compact_int8": (_i32, [_vp, _vp, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "kvz_decode_workspace_size": (_sz, [_i64, _i32, _i64, _i32]),
    "kvz_decode": (_i32, [_vp, _vp, _vp, _i64, _vp, _vp, _i64, _i32, _i64, _i32, _f32, _vp, _vp, _vp, _sz, _vp, _vp]),
    "kvz_head_score": (_i32, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "kvz_select_heads_workspace_size": (_sz, [_i64]),
    "kvz_select_heads": (_i32, [_vp, _i64, _i64, _f64, _vp, _i64, _vp, _vp, _vp, _sz, _vp, _vp]),
    "kvz_score_chunked_workspace_size": (_sz, [_i64, _i32, _i64, _i64, _i64]),
    "kvz_score_chunked": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i32, _i64, _i64, _i64, _i32, _f32, _vp, _vp, _sz,
                                 _vp, _vp]),
    "kvz_compress_host_workspace_size": (_sz, [_i64, _i32, _i64, _i64, _i32, _f64, _i32]),
    "kvz_compress_host": (_i32, [_vp, _vp, _vp, _vp, _i64, _i32, _i64, _i64, _i32, _f32, _f64, _i32, _vp, _i64,
                                 _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp, _vp]),
    "kvz_testing_compact_in_place_withhold": (_i32, [_vp, _vp, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _sz, _i64, _i64,
                                                     _i64, _vp, _vp]),
}


def lib():
    """The loaded libkvz.so (ctypes), with argument types declared."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise KvzLibraryError("libkvz.so not built (%s); run "
                                  "`python -m query_agnostic_kv_kvz_b200.build`" % lib_path)
        try:
            handle = ctypes.CDLL(lib_path)
        except OSError as e:  # pragma: no cover - depends on the machine
            raise KvzLibraryError("cannot load %s: %s" % (lib_path, e)) from e
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn: str, code: int):
    if code != 0:
        raise KvzError(fn, code)


def _req(fn: str, name: str, t, dtype=None, shape=None, ndim=None, numel=None):
    """Check one tensor argument before anything reaches the C ABI (which
    trusts the sizes it is given): type, dtype, dense layout, exact shape or
    rank, and a minimum element count.  ``None`` (an optional argument that
    was not passed) is accepted."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise ValueError("%s: %s must be a torch.Tensor" % (fn, name))
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s: %s must be %s, got %s" % (fn, name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s: %s must be contiguous" % (fn, name))
    if shape is not None and tuple(t.shape) != tuple(int(s) for s in shape):
        raise ValueError("%s: %s must have shape %s, got %s" % (fn, name, tuple(shape), tuple(t.shape)))
    if ndim is not None and t.dim() != ndim:
        raise ValueError("%s: %s must have %d dimensions, got %d" % (fn, name, ndim, t.dim()))
    if numel is not None and t.numel() < numel:
        raise ValueError("%s: %s holds %d elements, needs at least %d" % (fn, name, t.numel(), numel))


def _device(fn: str, *ts) -> torch.device:
    """The one CUDA device every given tensor lives on."""
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("%s: tensors must live on a CUDA device" % fn)
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("%s: tensors are on different devices (%s, %s)" % (fn, dev, t.device))
    if dev is None:
        raise ValueError("%s: no CUDA tensor given" % fn)
    return dev


def _status(fn: str, status):
    _req(fn, "status", status, torch.int32, numel=1)


def _bytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()




def kvz_version() -> int:
    return lib().kvz_version()


def kvz_keep_count(n: int, ratio: float) -> int:
    return lib().kvz_keep_count(int(n), float(ratio))


def kvz_score_workspace_size(B: int, G: int, n_in: int, row_chunk: int = 0) -> int:
    return lib().kvz_score_workspace_size(B, G, n_in, row_chunk)


def _score_shapes(fn, Q, K_ctx, K_in=None):
    _req(fn, "Q", Q, torch.bfloat16, ndim=4)
    _req(fn, "K_ctx", K_ctx, torch.bfloat16, ndim=3)
    B, G, n_in, d = Q.shape
    n_c = K_ctx.shape[1]
    if tuple(K_ctx.shape) != (B, n_c, d):
        raise ValueError("%s: K_ctx must be [B, n_c, d] = [%d, n_c, %d], got %s" % (fn, B, d, tuple(K_ctx.shape)))
    if K_in is not None:
        _req(fn, "K_in", K_in, torch.bfloat16, shape=(B, n_in, d))
    return B, G, n_in, d, n_c


def kvz_score(Q, K_ctx, K_in, scale: Optional[float] = None, row_chunk: int = 0, S=None, workspace=None,
              status=None, stream=None):
    """S[b, j] = max_{g,i} Softmax_causal(scale * Q_b K_b^T)[g, i, j] (KVzip §3.2); returns S."""
    fn = "kvz_score"
    if K_in is None:
        raise ValueError("%s: K_in is required" % fn)
    B, G, n_in, d, n_c = _score_shapes(fn, Q, K_ctx, K_in)
    _req(fn, "S", S, torch.float32, shape=(B, n_c))
    _req(fn, "workspace", workspace, torch.uint8)
    _status(fn, status)
    dev = _device(fn, Q, K_ctx, K_in, S, workspace, status)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(dev):
        if S is None:
            S = torch.empty((B, n_c), dtype=torch.float32, device=dev)
        if workspace is None:
            need = kvz_score_workspace_size(B, G, n_in, row_chunk)
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        _check(fn, lib().kvz_score(_ptr(Q), _ptr(K_ctx), _ptr(K_in), B, G, n_c, n_in, d, scale, row_chunk, _ptr(S),
                                   _ptr(workspace), _bytes(workspace), _ptr(status), _stream(stream)))
    return S


def kvz_score_noalloc(Q, K_ctx, K_in, scale: Optional[float] = None, S=None, status=None, stream=None):
    """kvz_score without a workspace, for callers that cannot allocate device
    memory at the point where they score.  The library's fixed static
    scratch is used instead (its size and sharing rules are in kvz.h); this
    wrapper allocates only S, and only when the caller passes none.  Calls
    that overlap on the GPU share that scratch and race."""
    fn = "kvz_score_noalloc"
    if K_in is None:
        raise ValueError("%s: K_in is required" % fn)
    B, G, n_in, d, n_c = _score_shapes(fn, Q, K_ctx, K_in)
    _req(fn, "S", S, torch.float32, shape=(B, n_c))
    _status(fn, status)
    dev = _device(fn, Q, K_ctx, K_in, S, status)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(dev):          # the static scratch and the stream are the tensors' device's
        if S is None:
            S = torch.empty((B, n_c), dtype=torch.float32, device=dev)
        _check(fn, lib().kvz_score_noalloc(_ptr(Q), _ptr(K_ctx), _ptr(K_in), B, G, n_c, n_in, d, scale, _ptr(S),
                                           _ptr(status), _stream(stream)))
    return S


def kvz_score_lse2(Q, K_ctx, K_in, i_begin: int = 0, i_end: Optional[int] = None, scale: Optional[float] = None,
                   lse2=None, ld: Optional[int] = None, workspace=None, status=None, stream=None):
    """Pass 1: base-2 log-sum-exp of input rows [i_begin, i_end); returns lse2 [B, G, ld].
    ``workspace`` (uint8, kvz_score_lse2_workspace_size() bytes) lets the
    grid's last wave be split over key ranges; it is allocated when not
    given."""
    fn = "kvz_score_lse2"
    if K_in is None:
        raise ValueError("%s: K_in is required" % fn)
    B, G, n_in, d, n_c = _score_shapes(fn, Q, K_ctx, K_in)
    i_end = n_in if i_end is None else int(i_end)
    if not (0 <= i_begin < i_end <= n_in) or i_begin % 256 != 0:
        raise ValueError("%s: need 0 <= i_begin < i_end <= n_in and i_begin %% 256 == 0" % fn)
    rows_pad = (i_end - i_begin + 255) // 256 * 256
    if lse2 is not None:
        _req(fn, "lse2", lse2, torch.float32, ndim=3)
        if tuple(lse2.shape[:2]) != (B, G):
            raise ValueError("%s: lse2 must be [B, G, ld]" % fn)
        ld = lse2.shape[2] if ld is None else int(ld)
        if ld != lse2.shape[2]:
            raise ValueError("%s: ld must equal lse2.shape[2]" % fn)
    ld = rows_pad if ld is None else int(ld)
    if ld < rows_pad or ld % 4 != 0:
        raise ValueError("%s: ld must be >= %d and a multiple of 4" % (fn, rows_pad))
    _req(fn, "workspace", workspace, torch.uint8)
    _status(fn, status)
    dev = _device(fn, Q, K_ctx, K_in, lse2, workspace, status)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(dev):
        if lse2 is None:
            lse2 = torch.empty((B, G, ld), dtype=torch.float32, device=dev)
        if workspace is None:
            workspace = torch.empty(kvz_score_lse2_workspace_size(), dtype=torch.uint8, device=dev)
        _check(fn, lib().kvz_score_lse2(_ptr(Q), _ptr(K_ctx), _ptr(K_in), B, G, n_c, n_in, d, scale, i_begin, i_end,
                                        _ptr(lse2), ld, _ptr(workspace), _bytes(workspace), _ptr(status),
                                        _stream(stream)))
    return lse2


def kvz_score_lse2_workspace_size() -> int:
    return lib().kvz_score_lse2_workspace_size()


def kvz_score_colmax(Q, K_ctx, lse2, i_begin: int = 0, i_end: Optional[int] = None,
                     scale: Optional[float] = None, S=None, accumulate: bool = False, status=None, stream=None):
    """Pass 2: context-key column max given pass 1's lse2 [B, G, ld]; returns S [B, n_c]."""
    fn = "kvz_score_colmax"
    B, G, n_in, d, n_c = _score_shapes(fn, Q, K_ctx)
    i_end = n_in if i_end is None else int(i_end)
    if not (0 <= i_begin < i_end <= n_in) or i_begin % 256 != 0:
        raise ValueError("%s: need 0 <= i_begin < i_end <= n_in and i_begin %% 256 == 0" % fn)
    rows_pad = (i_end - i_begin + 255) // 256 * 256
    _req(fn, "lse2", lse2, torch.float32, ndim=3)
    if tuple(lse2.shape[:2]) != (B, G) or lse2.shape[2] < rows_pad or lse2.shape[2] % 4 != 0:
        raise ValueError("%s: lse2 must be [B, G, ld] with ld >= %d, ld %% 4 == 0" % (fn, rows_pad))
    _req(fn, "S", S, torch.float32, shape=(B, n_c))
    if accumulate and S is None:
        raise ValueError("%s: accumulate needs the S to merge into" % fn)
    _status(fn, status)
    dev = _device(fn, Q, K_ctx, lse2, S, status)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(dev):
        if S is None:
            S = torch.empty((B, n_c), dtype=torch.float32, device=dev)
        ld = lse2.shape[-1]
        _check(fn, lib().kvz_score_colmax(_ptr(Q), _ptr(K_ctx), B, G, n_c, n_in, d, scale, i_begin, i_end,
                                          _ptr(lse2), ld, _ptr(S), int(bool(accumulate)), _ptr(status),
                                          _stream(stream)))
    return S


def kvz_select_workspace_size(B: int, n_c: int, mode: int) -> int:
    return lib().kvz_select_workspace_size(B, n_c, mode)


def _mode(mode) -> int:
    if mode in ("per_head", PER_HEAD):
        return PER_HEAD
    if mode in ("global", GLOBAL):
        return GLOBAL
    raise ValueError("mode must be 'per_head' or 'global'")


def _keep(n: int, ratio: float) -> int:
    """floor(ratio * n) with the product in IEEE double (kvz_keep_count)."""
    ratio = float(ratio)
    if not (0.0 <= ratio <= 1.0):
        raise ValueError("ratio must lie in [0, 1]")
    return int(math.floor(ratio * float(n)))


def _csr_args(fn, B, idx, counts, offsets, idx_min=None):
    _req(fn, "idx", idx, torch.int32, ndim=1, numel=idx_min)
    _req(fn, "counts", counts, torch.int32, numel=B)
    _req(fn, "offsets", offsets, torch.int64, numel=B + 1)


def _scores_2d(fn, S, name="S"):
    if S is None:
        raise ValueError("%s: %s is required" % (fn, name))
    _req(fn, name, S, torch.float32, ndim=2)
    return S.shape[0], S.shape[1]


def kvz_select(S, ratio: float, mode="per_head", idx=None, counts=None, offsets=None, workspace=None,
               status=None, stream=None):
    """Top-ratio selection (KVzip §4.1); returns (idx int32, counts int32 [B], offsets int64 [B+1])."""
    fn = "kvz_select"
    B, n_c = _scores_2d(fn, S)
    m = _mode(mode)
    k = _keep(B * n_c if m == GLOBAL else n_c, ratio)
    cap = k if m == GLOBAL else B * k
    _csr_args(fn, B, idx, counts, offsets, idx_min=cap)
    _req(fn, "workspace", workspace, torch.uint8)
    _status(fn, status)
    dev = _device(fn, S, idx, counts, offsets, workspace, status)
    with torch.cuda.device(dev):
        if idx is None:
            idx = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
        if counts is None:
            counts = torch.empty(B, dtype=torch.int32, device=dev)
        if offsets is None:
            offsets = torch.empty(B + 1, dtype=torch.int64, device=dev)
        if workspace is None:
            need = kvz_select_workspace_size(B, n_c, m)
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        _check(fn, lib().kvz_select(_ptr(S), B, n_c, float(ratio), m, _ptr(idx), idx.numel(), _ptr(counts),
                                    _ptr(offsets), _ptr(workspace), _bytes(workspace), _ptr(status),
                                    _stream(stream)))
    return idx, counts, offsets


def kvz_select_dist_workspace_size(B_local: int, n_c: int) -> int:
    return lib().kvz_select_dist_workspace_size(B_local, n_c)


def _dist_args(fn, S, hist, workspace):
    B, n_c = _scores_2d(fn, S)
    _req(fn, "hist", hist, ndim=1, numel=2048)
    if hist is not None and hist.element_size() != 4:
        raise ValueError("%s: hist must hold 32-bit bins" % fn)
    if workspace is None:
        raise ValueError("%s: workspace is required (it carries the state between calls)" % fn)
    _req(fn, "workspace", workspace, torch.uint8)
    return B, n_c


def kvz_select_dist_begin(S, B_total: int, ratio: float, hist, workspace, status=None, stream=None):
    """First step of the global selection over heads split across ranks:
    this rank's first-digit histogram into hist (uint32 [2048], as int32)."""
    fn = "kvz_select_dist_begin"
    B, n_c = _dist_args(fn, S, hist, workspace)
    _status(fn, status)
    dev = _device(fn, S, hist, workspace, status)
    with torch.cuda.device(dev):
        _check(fn, lib().kvz_select_dist_begin(_ptr(S), B, n_c, int(B_total), float(ratio), _ptr(hist),
                                               _ptr(workspace), _bytes(workspace), _ptr(status), _stream(stream)))


def kvz_select_dist_step(S, pass_: int, hist, eq_total, workspace, status=None, stream=None):
    """Digit pick from the rank-summed hist; the next local histogram, or
    (pass 2) this rank's threshold-equal count into eq_total (int64 [1])."""
    fn = "kvz_select_dist_step"
    B, n_c = _dist_args(fn, S, hist, workspace)
    _req(fn, "eq_total", eq_total, torch.int64, numel=1)
    if int(pass_) == 2 and eq_total is None:
        raise ValueError("%s: pass 2 writes eq_total" % fn)
    _status(fn, status)
    dev = _device(fn, S, hist, eq_total, workspace, status)
    with torch.cuda.device(dev):
        _check(fn, lib().kvz_select_dist_step(_ptr(S), B, n_c, int(pass_), _ptr(hist), _ptr(eq_total),
                                              _ptr(workspace), _bytes(workspace), _ptr(status), _stream(stream)))


def kvz_select_dist_finish(S, B_total: int, ratio: float, eq_ranks, rank: int, idx, counts, offsets, workspace,
                           status=None, stream=None):
    """Last step: this rank's kept positions (CSR over its own heads)."""
    fn = "kvz_select_dist_finish"
    B, n_c = _scores_2d(fn, S)
    _req(fn, "eq_ranks", eq_ranks, torch.int64, ndim=1, numel=int(rank) + 1)
    k = _keep(int(B_total) * n_c, ratio)
    if idx is None or counts is None or offsets is None:
        raise ValueError("%s: idx, counts and offsets are required" % fn)
    _csr_args(fn, B, idx, counts, offsets, idx_min=min(k, B * n_c))
    if workspace is None:
        raise ValueError("%s: workspace is required" % fn)
    _req(fn, "workspace", workspace, torch.uint8)
    _status(fn, status)
    dev = _device(fn, S, eq_ranks, idx, counts, offsets, workspace, status)
    with torch.cuda.device(dev):
        _check(fn, lib().kvz_select_dist_finish(_ptr(S), B, n_c, int(B_total), float(ratio), _ptr(eq_ranks),
                                                int(rank), _ptr(idx), idx.numel(), _ptr(counts), _ptr(offsets),
                                                _ptr(workspace), _bytes(workspace), _ptr(status), _stream(stream)))


def kvz_compact_workspace_size(B: int, n_c: int) -> int:
    return lib().kvz_compact_workspace_size(B, n_c)


def _kv_pair(fn, K, V):
    _req(fn, "K", K, torch.bfloat16, ndim=3)
    _req(fn, "V", V, torch.bfloat16, ndim=3)
    if K is None or V is None or K.shape != V.shape:
        raise ValueError("%s: K and V must be bfloat16 [B, n_c, d] of equal shape" % fn)
    return K.shape


def _rows_out(fn, name, t, dtype, d, min_rows):
    _req(fn, name, t, dtype, ndim=2)
    if t is not None and (t.shape[1] != d or t.shape[0] < min_rows):
        raise ValueError("%s: %s must be [rows >= %d, %d], got %s" % (fn, name, min_rows, d, tuple(t.shape)))


def kvz_compact(K, V, idx, counts, offsets, out_offsets=None, K_out=None, V_out=None, in_place: bool = False,
                out_rows: Optional[int] = None, workspace=None, status=None, stream=None):
    """Gather kept rows in key order (KVzip §2.1 pruned cache); returns (K_out, V_out).

    Out of place, the outputs are [rows, d] with head b's rows starting at
    out_offsets[b] (default offsets[b]); ``out_rows`` sizes freshly allocated
    outputs (default B*n_c, an upper bound).  A packed output (no
    out_offsets) must have at least min(idx.numel(), B*n_c) rows, the most a
    selection into that idx can keep; with out_offsets the caller guarantees
    room for out_offsets[b] + counts[b] rows.  In place, K and V themselves
    are returned, each head's kept rows packed to the front of its region.
    """
    fn = "kvz_compact"
    B, n_c, d = _kv_pair(fn, K, V)
    if idx is None or counts is None or offsets is None:
        raise ValueError("%s: idx, counts and offsets are required" % fn)
    _csr_args(fn, B, idx, counts, offsets)
    _req(fn, "out_offsets", out_offsets, torch.int64, numel=B)
    _req(fn, "workspace", workspace, torch.uint8)
    _status(fn, status)
    if in_place:
        if out_offsets is not None or K_out is not None or V_out is not None:
            raise ValueError("%s: in place takes no out_offsets, K_out or V_out" % fn)
    else:
        min_rows = 0 if out_offsets is not None else min(idx.numel(), B * n_c)
        if out_rows is not None and int(out_rows) < min_rows:
            raise ValueError("%s: out_rows must be >= %d" % (fn, min_rows))
        _rows_out(fn, "K_out", K_out, torch.bfloat16, d, min_rows)
        _rows_out(fn, "V_out", V_out, torch.bfloat16, d, min_rows)
    dev = _device(fn, K, V, idx, counts, offsets, out_offsets, K_out, V_out, workspace, status)
    with torch.cuda.device(dev):
        if in_place:
            K_out, V_out = K, V
            if workspace is None:
                workspace = torch.empty(kvz_compact_workspace_size(B, n_c), dtype=torch.uint8, device=dev)
        else:
            rows = B * n_c if out_rows is None else int(out_rows)
            if K_out is None:
                K_out = torch.empty((rows, d), dtype=K.dtype, device=dev)
            if V_out is None:
                V_out = torch.empty((rows, d), dtype=V.dtype, device=dev)
        _check(fn, lib().kvz_compact(_ptr(K), _ptr(V), B, n_c, d, _ptr(idx), _ptr(counts), _ptr(offsets),
                                     _ptr(out_offsets), _ptr(K_out), _ptr(V_out), _ptr(workspace),
                                     _bytes(workspace), _ptr(status), _stream(stream)))
    return K_out, V_out


def kvz_compress_host_workspace_size(B: int, G: int, n_c: int, n_in: int, d: int, ratio: float, mode) -> int:
    return lib().kvz_compress_host_workspace_size(B, G, n_c, n_in, d, float(ratio), _mode(mode))


def kvz_compress_host(Q, K_ctx, K_in, V, ratio: float, mode="per_head", scale: Optional[float] = None, out=None,
                      workspace=None, status=None, stream=None, copy_stream=None):
    """The whole path of one context from host tensors to host tensors
    (score, select, out-of-place compact); returns a dict with ``idx``,
    ``counts``, ``offsets``, ``K_out`` and ``V_out`` (CPU tensors, valid once
    ``stream`` has finished).  Inputs should be page-locked for the copies to
    overlap the scoring; ``out`` may pass preallocated (pinned) outputs."""
    fn = "kvz_compress_host"
    for name, t in (("Q", Q), ("K_ctx", K_ctx), ("K_in", K_in), ("V", V)):
        if t is None or t.is_cuda:
            raise ValueError("%s: %s must be a CPU tensor" % (fn, name))
        _req(fn, name, t, torch.bfloat16)
    if Q.dim() != 4:
        raise ValueError("%s: Q must be [B, G, n_in, d]" % fn)
    B, G, n_in, d = Q.shape
    n_c = K_ctx.shape[1] if K_ctx.dim() == 3 else -1
    if K_ctx.shape != (B, n_c, d) or V.shape != (B, n_c, d) or K_in.shape != (B, n_in, d):
        raise ValueError("%s: shapes must be Q [B,G,n_in,d], K_ctx/V [B,n_c,d], K_in [B,n_in,d]" % fn)
    m = _mode(mode)
    k = _keep(B * n_c if m == GLOBAL else n_c, ratio)
    kept = k if m == GLOBAL else B * k
    if out is not None:
        for name, dt, n in (("idx", torch.int32, kept), ("counts", torch.int32, B), ("offsets", torch.int64, B + 1)):
            t = out.get(name)
            if t is None or t.is_cuda:
                raise ValueError("%s: out[%r] must be a CPU tensor" % (fn, name))
            _req(fn, "out[%r]" % name, t, dt, numel=n)
        for name in ("K_out", "V_out"):
            t = out.get(name)
            if t is None or t.is_cuda:
                raise ValueError("%s: out[%r] must be a CPU tensor" % (fn, name))
            _rows_out(fn, "out[%r]" % name, t, torch.bfloat16, d, kept)
    _req(fn, "workspace", workspace, torch.uint8)
    _status(fn, status)
    dev = _device(fn, workspace, status) if (workspace is not None or status is not None) else \
        torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        if out is None:
            pin = Q.is_pinned()
            out = {"idx": torch.empty(max(kept, 1), dtype=torch.int32, pin_memory=pin),
                   "counts": torch.empty(B, dtype=torch.int32, pin_memory=pin),
                   "offsets": torch.empty(B + 1, dtype=torch.int64, pin_memory=pin),
                   "K_out": torch.empty((max(kept, 1), d), dtype=torch.bfloat16, pin_memory=pin),
                   "V_out": torch.empty((max(kept, 1), d), dtype=torch.bfloat16, pin_memory=pin)}
        if workspace is None:
            workspace = torch.empty(kvz_compress_host_workspace_size(B, G, n_c, n_in, d, ratio, m),
                                    dtype=torch.uint8, device=dev)
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        st = _stream(stream)
        cst = _stream(copy_stream) if copy_stream is not None else st
        _check(fn, lib().kvz_compress_host(
            _ptr(Q), _ptr(K_ctx), _ptr(K_in), _ptr(V), B, G, n_c, n_in, d, float(scale), float(ratio), m,
            _ptr(out["idx"]), out["idx"].numel(), _ptr(out["counts"]), _ptr(out["offsets"]), _ptr(out["K_out"]),
            _ptr(out["V_out"]), _ptr(workspace), _bytes(workspace), _ptr(status), st, cst))
    return out


def kvz_score_chunked_workspace_size(B: int, G: int, n_c: int, n_prompt: int, m: int) -> int:
    return lib().kvz_score_chunked_workspace_size(B, G, n_c, n_prompt, m)


def kvz_score_chunked(Q, Q_tail, K_ctx, K_in, K_in_tail, m: int, scale: Optional[float] = None, S=None,
                      workspace=None, status=None, stream=None):
    """Chunked importance scores (KVzip §3.4); returns S [B, n_c] fp32.

    Q [B, T, G, n_prompt+m, d] and K_in [B, T, n_prompt+m, d] hold the T full
    chunks' inputs, Q_tail / K_in_tail the shorter last chunk's (None when m
    divides n_c); K_ctx is [B, n_c, d]."""
    fn = "kvz_score_chunked"
    _req(fn, "K_ctx", K_ctx, torch.bfloat16, ndim=3)
    if K_ctx is None:
        raise ValueError("%s: K_ctx is required" % fn)
    B, n_c, d = K_ctx.shape
    m = int(m)
    if m < 1:
        raise ValueError("%s: m must be >= 1" % fn)
    T, m_last = n_c // m, n_c % m
    ref = Q if Q is not None else Q_tail
    if ref is None or ref.dim() < 3:
        raise ValueError("%s: Q (or Q_tail) is required" % fn)
    G = ref.shape[-3]
    n_prompt = (Q.shape[-2] - m) if Q is not None else (Q_tail.shape[-2] - m_last)
    if n_prompt < 0:
        raise ValueError("%s: the query rows must hold n_prompt + m_t >= m_t tokens" % fn)
    if T > 0:
        _req(fn, "Q", Q, torch.bfloat16, shape=(B, T, G, n_prompt + m, d))
        _req(fn, "K_in", K_in, torch.bfloat16, shape=(B, T, n_prompt + m, d))
        if Q is None or K_in is None:
            raise ValueError("%s: Q must be [B, T, G, n_prompt+m, d] and K_in [B, T, n_prompt+m, d]" % fn)
    if m_last > 0:
        _req(fn, "Q_tail", Q_tail, torch.bfloat16, shape=(B, G, n_prompt + m_last, d))
        _req(fn, "K_in_tail", K_in_tail, torch.bfloat16, shape=(B, n_prompt + m_last, d))
        if Q_tail is None or K_in_tail is None:
            raise ValueError("%s: Q_tail must be [B, G, n_prompt+m_last, d] and K_in_tail "
                             "[B, n_prompt+m_last, d]" % fn)
    _req(fn, "S", S, torch.float32, shape=(B, n_c))
    _req(fn, "workspace", workspace, torch.uint8)
    _status(fn, status)
    dev = _device(fn, Q, Q_tail, K_ctx, K_in, K_in_tail, S, workspace, status)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(dev):
        if S is None:
            S = torch.empty((B, n_c), dtype=torch.float32, device=dev)
        if workspace is None:
            workspace = torch.empty(kvz_score_chunked_workspace_size(B, G, n_c, n_prompt, m), dtype=torch.uint8,
                                    device=dev)
        _check(fn, lib().kvz_score_chunked(
            _ptr(Q), _ptr(Q_tail), _ptr(K_ctx), _ptr(K_in), _ptr(K_in_tail), B, G, n_c, n_prompt, m, d,
            float(scale), _ptr(S), _ptr(workspace), _bytes(workspace), _ptr(status), _stream(stream)))
    return S


def kvz_head_score(S, S_head=None, status=None, stream=None):
    """Context-independent head scores (KVzip §4.2): S_head[b] = max_j S[b, j]."""
    fn = "kvz_head_score"
    B, n_c = _scores_2d(fn, S)
    _req(fn, "S_head", S_head, torch.float32, numel=B)
    _status(fn, status)
    dev = _device(fn, S, S_head, status)
    with torch.cuda.device(dev):
        if S_head is None:
            S_head = torch.empty(B, dtype=torch.float32, device=dev)
        _check(fn, lib().kvz_head_score(_ptr(S), B, n_c, _ptr(S_head), _ptr(status), _stream(stream)))
    return S_head


def kvz_select_heads(S_head, n_c: int, ratio: float, idx=None, counts=None, offsets=None, workspace=None,
                     status=None, stream=None):
    """Head-level eviction: keep the floor(ratio*B) best heads whole; returns
    (idx, counts, offsets) in kvz_select's form, ready for kvz_compact."""
    fn = "kvz_select_heads"
    if S_head is None:
        raise ValueError("%s: S_head is required" % fn)
    _req(fn, "S_head", S_head, torch.float32, ndim=1)
    B = S_head.shape[0]
    n_c = int(n_c)
    if n_c < 1:
        raise ValueError("%s: n_c must be >= 1" % fn)
    k = _keep(B, ratio)
    _csr_args(fn, B, idx, counts, offsets, idx_min=k * n_c)
    _req(fn, "workspace", workspace, torch.uint8)
    _status(fn, status)
    dev = _device(fn, S_head, idx, counts, offsets, workspace, status)
    with torch.cuda.device(dev):
        if idx is None:
            idx = torch.empty(max(1, k * n_c), dtype=torch.int32, device=dev)
        if counts is None:
            counts = torch.empty(B, dtype=torch.int32, device=dev)
        if offsets is None:
            offsets = torch.empty(B + 1, dtype=torch.int64, device=dev)
        if workspace is None:
            workspace = torch.empty(lib().kvz_select_heads_workspace_size(B), dtype=torch.uint8, device=dev)
        _check(fn, lib().kvz_select_heads(_ptr(S_head), B, n_c, float(ratio), _ptr(idx), idx.numel(), _ptr(counts),
                                          _ptr(offsets), _ptr(workspace), _bytes(workspace), _ptr(status),
                                          _stream(stream)))
    return idx, counts, offsets


def kvz_decode(q, K_out, V_out, counts, offsets, n_c: int, scale: Optional[float] = None, out=None, lse2=None,
               workspace=None, status=None, stream=None):
    """One decode step of attention over the pruned cache; returns (out [B, G, d]
    fp32, lse2 [B, G] fp32).  q is bf16 [B, G, d]; K_out / V_out are the packed
    [rows, d] caches kvz_compact writes; n_c bounds every head's count."""
    fn = "kvz_decode"
    _req(fn, "q", q, torch.bfloat16, ndim=3)
    if q is None:
        raise ValueError("%s: q is required" % fn)
    B, G, d = q.shape
    _rows_out(fn, "K_out", K_out, torch.bfloat16, d, 1)
    _rows_out(fn, "V_out", V_out, torch.bfloat16, d, 1)
    if K_out is None or V_out is None or K_out.shape != V_out.shape:
        raise ValueError("%s: K_out and V_out must be bfloat16 [rows, d] of equal shape" % fn)
    if counts is None or offsets is None:
        raise ValueError("%s: counts and offsets are required" % fn)
    _csr_args(fn, B, None, counts, offsets)
    _req(fn, "out", out, torch.float32, shape=(B, G, d))
    _req(fn, "lse2", lse2, torch.float32, shape=(B, G))
    _req(fn, "workspace", workspace, torch.uint8)
    _status(fn, status)
    dev = _device(fn, q, K_out, V_out, counts, offsets, out, lse2, workspace, status)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(dev):
        if out is None:
            out = torch.empty((B, G, d), dtype=torch.float32, device=dev)
        if lse2 is None:
            lse2 = torch.empty((B, G), dtype=torch.float32, device=dev)
        if workspace is None:
            workspace = torch.empty(max(1, lib().kvz_decode_workspace_size(B, G, n_c, d)), dtype=torch.uint8,
                                    device=dev)
        _check(fn, lib().kvz_decode(_ptr(q), _ptr(K_out), _ptr(V_out), K_out.shape[0], _ptr(counts), _ptr(offsets),
                                    B, G, int(n_c), d, float(scale), _ptr(out), _ptr(lse2), _ptr(workspace),
                                    _bytes(workspace), _ptr(status), _stream(stream)))
    return out, lse2


def kvz_select_protected(S, ratio: float, mode="per_head", n_protect: int = 0, idx=None, counts=None, offsets=None,
                         workspace=None, status=None, stream=None):
    """kvz_select with the first n_protect positions of every head always
    kept (KVzip §4.1 system prompt); the ratio applies to the rest."""
    fn = "kvz_select_protected"
    B, n_c = _scores_2d(fn, S)
    m = _mode(mode)
    n_protect = int(n_protect)
    if not (0 <= n_protect <= n_c):
        raise ValueError("%s: need 0 <= n_protect <= n_c" % fn)
    free = n_c - n_protect
    k = (B * n_protect + _keep(B * free, ratio)) if m == GLOBAL else (n_protect + _keep(free, ratio))
    cap = k if m == GLOBAL else B * k
    _csr_args(fn, B, idx, counts, offsets, idx_min=cap)
    _req(fn, "workspace", workspace, torch.uint8)
    _status(fn, status)
    dev = _device(fn, S, idx, counts, offsets, workspace, status)
    with torch.cuda.device(dev):
        if idx is None:
            idx = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
        if counts is None:
            counts = torch.empty(B, dtype=torch.int32, device=dev)
        if offsets is None:
            offsets = torch.empty(B + 1, dtype=torch.int64, device=dev)
        if workspace is None:
            workspace = torch.empty(kvz_select_workspace_size(B, n_c, m), dtype=torch.uint8, device=dev)
        _check(fn, lib().kvz_select_protected(_ptr(S), B, n_c, float(ratio), m, n_protect, _ptr(idx), idx.numel(),
                                              _ptr(counts), _ptr(offsets), _ptr(workspace), _bytes(workspace),
                                              _ptr(status), _stream(stream)))
    return idx, counts, offsets


def kvz_compact_int8(K, V, idx, counts, offsets, out_offsets=None, out_rows: Optional[int] = None, Kq=None, Vq=None,
                     K_scale=None, V_scale=None, status=None, stream=None):
    """Out-of-place compaction into int8 codes with one fp32 scale per row
    (KVzip §4.2 KV quantisation); returns (Kq, K_scale, Vq, V_scale).  Row
    capacity rules are kvz_compact's: a packed output (no out_offsets) needs
    at least min(idx.numel(), B*n_c) rows in every output."""
    fn = "kvz_compact_int8"
    B, n_c, d = _kv_pair(fn, K, V)
    if idx is None or counts is None or offsets is None:
        raise ValueError("%s: idx, counts and offsets are required" % fn)
    _csr_args(fn, B, idx, counts, offsets)
    _req(fn, "out_offsets", out_offsets, torch.int64, numel=B)
    min_rows = 0 if out_offsets is not None else min(idx.numel(), B * n_c)
    if out_rows is not None and int(out_rows) < min_rows:
        raise ValueError("%s: out_rows must be >= %d" % (fn, min_rows))
    _rows_out(fn, "Kq", Kq, torch.int8, d, min_rows)
    _rows_out(fn, "Vq", Vq, torch.int8, d, min_rows)
    rows = int(out_rows) if out_rows is not None else (Kq.shape[0] if Kq is not None else B * n_c)
    _req(fn, "K_scale", K_scale, torch.float32, ndim=1, numel=Kq.shape[0] if Kq is not None else rows)
    _req(fn, "V_scale", V_scale, torch.float32, ndim=1, numel=Vq.shape[0] if Vq is not None else rows)
    _status(fn, status)
    dev = _device(fn, K, V, idx, counts, offsets, out_offsets, Kq, Vq, K_scale, V_scale, status)
    with torch.cuda.device(dev):
        Kq = torch.empty((rows, d), dtype=torch.int8, device=dev) if Kq is None else Kq
        Vq = torch.empty((rows, d), dtype=torch.int8, device=dev) if Vq is None else Vq
        K_scale = torch.empty(Kq.shape[0], dtype=torch.float32, device=dev) if K_scale is None else K_scale
        V_scale = torch.empty(Vq.shape[0], dtype=torch.float32, device=dev) if V_scale is None else V_scale
        _check(fn, lib().kvz_compact_int8(_ptr(K), _ptr(V), B, n_c, d, _ptr(idx), _ptr(counts), _ptr(offsets),
                                          _ptr(out_offsets), _ptr(Kq), _ptr(Vq), _ptr(K_scale), _ptr(V_scale),
                                          _ptr(status), _stream(stream)))
    return Kq, K_scale, Vq, V_scale


def kvz_testing_compact_in_place_withhold(K, V, idx, counts, offsets, wait_ns: int, hold_head: int,
                                          hold_chunk: int, workspace=None, status=None, stream=None):
    """Test-only (include/kvz_testing.h): in-place kvz_compact whose ordering
    waits give up after ``wait_ns`` and whose chunk ``hold_chunk`` of head
    ``hold_head`` never reports its sources read, so a chunk waiting on it
    times out with KVZ_ERR_TIMEOUT in ``status``.  Returns (K, V)."""
    fn = "kvz_testing_compact_in_place_withhold"
    B, n_c, d = _kv_pair(fn, K, V)
    if idx is None or counts is None or offsets is None:
        raise ValueError("%s: idx, counts and offsets are required" % fn)
    _csr_args(fn, B, idx, counts, offsets)
    _req(fn, "workspace", workspace, torch.uint8)
    _status(fn, status)
    dev = _device(fn, K, V, idx, counts, offsets, workspace, status)
    with torch.cuda.device(dev):
        if workspace is None:
            workspace = torch.empty(kvz_compact_workspace_size(B, n_c), dtype=torch.uint8, device=dev)
        _check(fn, lib().kvz_testing_compact_in_place_withhold(
            _ptr(K), _ptr(V), B, n_c, d, _ptr(idx), _ptr(counts), _ptr(offsets), _ptr(workspace), _bytes(workspace),
            int(wait_ns), int(hold_head), int(hold_chunk), _ptr(status), _stream(stream)))
    return K, V
