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
    "kvz_score_lse2", "kvz_score_colmax", "kvz_select_workspace_size", "kvz_select",
    "kvz_select_dist_workspace_size", "kvz_select_dist_begin", "kvz_select_dist_step", "kvz_select_dist_finish",
    "kvz_compact_workspace_size", "kvz_compact", "kvz_compress_host_workspace_size", "kvz_compress_host",
    "kvz_score_chunked_workspace_size", "kvz_score_chunked", "kvz_head_score", "kvz_select_heads", "kvz_decode",
    "kvz_select_protected", "kvz_compact_int8",
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
    "kvz_score_lse2": (_i32, [_vp, _vp, _vp, _i64, _i32, _i64, _i64, _i32, _f32, _i64, _i64, _vp, _i64, _vp,
                              _vp]),
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


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("kvz: tensors must live on a CUDA device")


def kvz_version() -> int:
    return lib().kvz_version()


def kvz_keep_count(n: int, ratio: float) -> int:
    return lib().kvz_keep_count(int(n), float(ratio))


def kvz_score_workspace_size(B: int, G: int, n_in: int, row_chunk: int = 0) -> int:
    return lib().kvz_score_workspace_size(B, G, n_in, row_chunk)


def _score_shapes(Q, K_ctx, K_in=None):
    if Q.dim() != 4 or K_ctx.dim() != 3:
        raise ValueError("expected Q[B,G,n_in,d] and K_ctx[B,n_c,d]")
    B, G, n_in, d = Q.shape
    if K_ctx.shape[0] != B or K_ctx.shape[2] != d:
        raise ValueError("K_ctx shape does not match Q")
    if K_in is not None and tuple(K_in.shape) != (B, n_in, d):
        raise ValueError("K_in must be [B, n_in, d]")
    for t in (Q, K_ctx, K_in):
        if t is not None and (t.dtype != torch.bfloat16 or not t.is_contiguous()):
            raise ValueError("Q/K must be contiguous bfloat16")
    return B, G, n_in, d, K_ctx.shape[1]


def kvz_score(Q, K_ctx, K_in, scale: Optional[float] = None, row_chunk: int = 0, S=None, workspace=None,
              status=None, stream=None):
    """S[b, j] = max_{g,i} Softmax_causal(scale * Q_b K_b^T)[g, i, j] (KVzip §3.2); returns S."""
    _need_cuda(Q, K_ctx, K_in, S, workspace, status)
    B, G, n_in, d, n_c = _score_shapes(Q, K_ctx, K_in)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if S is None:
        S = torch.empty((B, n_c), dtype=torch.float32, device=Q.device)
    need = kvz_score_workspace_size(B, G, n_in, row_chunk)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=Q.device)
    nbytes = workspace.numel() * workspace.element_size()
    _check("kvz_score", lib().kvz_score(_ptr(Q), _ptr(K_ctx), _ptr(K_in), B, G, n_c, n_in, d, scale, row_chunk,
                                        _ptr(S), _ptr(workspace), nbytes, _ptr(status), _stream(stream)))
    return S


def kvz_score_noalloc(Q, K_ctx, K_in, scale: Optional[float] = None, S=None, status=None, stream=None):
    """kvz_score without a workspace: for callers that cannot allocate device
    memory when they score.  The library's fixed static scratch is used
    instead (see include/kvz.h); only S is allocated here, and only when the
    caller passes none.  Calls that overlap on the GPU share that scratch."""
    _need_cuda(Q, K_ctx, K_in, S, status)
    B, G, n_in, d, n_c = _score_shapes(Q, K_ctx, K_in)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if S is None:
        S = torch.empty((B, n_c), dtype=torch.float32, device=Q.device)
    _check("kvz_score_noalloc", lib().kvz_score_noalloc(_ptr(Q), _ptr(K_ctx), _ptr(K_in), B, G, n_c, n_in, d,
                                                        scale, _ptr(S), _ptr(status), _stream(stream)))
    return S


def kvz_score_lse2(Q, K_ctx, K_in, i_begin: int = 0, i_end: Optional[int] = None, scale: Optional[float] = None,
                   lse2=None, ld: Optional[int] = None, status=None, stream=None):
    """Pass 1: base-2 log-sum-exp of input rows [i_begin, i_end); returns lse2 [B, G, ld]."""
    _need_cuda(Q, K_ctx, K_in, lse2, status)
    B, G, n_in, d, n_c = _score_shapes(Q, K_ctx, K_in)
    i_end = n_in if i_end is None else i_end
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rows_pad = (i_end - i_begin + 255) // 256 * 256
    ld = rows_pad if ld is None else ld
    if lse2 is None:
        lse2 = torch.empty((B, G, ld), dtype=torch.float32, device=Q.device)
    _check("kvz_score_lse2", lib().kvz_score_lse2(_ptr(Q), _ptr(K_ctx), _ptr(K_in), B, G, n_c, n_in, d, scale,
                                                  i_begin, i_end, _ptr(lse2), ld, _ptr(status), _stream(stream)))
    return lse2


def kvz_score_colmax(Q, K_ctx, lse2, i_begin: int = 0, i_end: Optional[int] = None,
                     scale: Optional[float] = None, S=None, accumulate: bool = False, status=None, stream=None):
    """Pass 2: context-key column max given pass 1's lse2 [B, G, ld]; returns S [B, n_c]."""
    _need_cuda(Q, K_ctx, lse2, S, status)
    B, G, n_in, d, n_c = _score_shapes(Q, K_ctx)
    i_end = n_in if i_end is None else i_end
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if S is None:
        S = torch.empty((B, n_c), dtype=torch.float32, device=Q.device)
    ld = lse2.shape[-1]
    _check("kvz_score_colmax", lib().kvz_score_colmax(_ptr(Q), _ptr(K_ctx), B, G, n_c, n_in, d, scale, i_begin,
                                                      i_end, _ptr(lse2), ld, _ptr(S), int(bool(accumulate)),
                                                      _ptr(status), _stream(stream)))
    return S


def kvz_select_workspace_size(B: int, n_c: int, mode: int) -> int:
    return lib().kvz_select_workspace_size(B, n_c, mode)


def _mode(mode) -> int:
    if mode in ("per_head", PER_HEAD):
        return PER_HEAD
    if mode in ("global", GLOBAL):
        return GLOBAL
    raise ValueError("mode must be 'per_head' or 'global'")


def kvz_select(S, ratio: float, mode="per_head", idx=None, counts=None, offsets=None, workspace=None,
               status=None, stream=None):
    """Top-ratio selection (KVzip §4.1); returns (idx int32, counts int32 [B], offsets int64 [B+1])."""
    _need_cuda(S, idx, counts, offsets, workspace, status)
    if S.dim() != 2 or S.dtype != torch.float32 or not S.is_contiguous():
        raise ValueError("S must be a contiguous float32 [B, n_c] tensor")
    m = _mode(mode)
    B, n_c = S.shape
    k = kvz_keep_count(B * n_c if m == GLOBAL else n_c, ratio)
    cap = k if m == GLOBAL else B * k
    if idx is None:
        idx = torch.empty(max(cap, 1), dtype=torch.int32, device=S.device)
    if counts is None:
        counts = torch.empty(B, dtype=torch.int32, device=S.device)
    if offsets is None:
        offsets = torch.empty(B + 1, dtype=torch.int64, device=S.device)
    need = kvz_select_workspace_size(B, n_c, m)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=S.device)
    nbytes = workspace.numel() * workspace.element_size()
    _check("kvz_select", lib().kvz_select(_ptr(S), B, n_c, float(ratio), m, _ptr(idx), idx.numel(), _ptr(counts),
                                          _ptr(offsets), _ptr(workspace), nbytes, _ptr(status), _stream(stream)))
    return idx, counts, offsets


def kvz_select_dist_workspace_size(B_local: int, n_c: int) -> int:
    return lib().kvz_select_dist_workspace_size(B_local, n_c)


def _dist_args(S, workspace):
    if S.dim() != 2 or S.dtype != torch.float32 or not S.is_contiguous():
        raise ValueError("S must be a contiguous float32 [B_local, n_c] tensor")
    return S.shape[0], S.shape[1], workspace.numel() * workspace.element_size()


def kvz_select_dist_begin(S, B_total: int, ratio: float, hist, workspace, status=None, stream=None):
    """First step of the global selection over heads split across ranks:
    this rank's first-digit histogram into hist (uint32 [2048], as int32)."""
    _need_cuda(S, hist, workspace, status)
    B, n_c, nbytes = _dist_args(S, workspace)
    _check("kvz_select_dist_begin", lib().kvz_select_dist_begin(
        _ptr(S), B, n_c, int(B_total), float(ratio), _ptr(hist), _ptr(workspace), nbytes, _ptr(status),
        _stream(stream)))


def kvz_select_dist_step(S, pass_: int, hist, eq_total, workspace, status=None, stream=None):
    """Digit pick from the rank-summed hist; the next local histogram, or
    (pass 2) this rank's threshold-equal count into eq_total (int64 [1])."""
    _need_cuda(S, hist, eq_total, workspace, status)
    B, n_c, nbytes = _dist_args(S, workspace)
    _check("kvz_select_dist_step", lib().kvz_select_dist_step(
        _ptr(S), B, n_c, int(pass_), _ptr(hist), _ptr(eq_total), _ptr(workspace), nbytes, _ptr(status),
        _stream(stream)))


def kvz_select_dist_finish(S, B_total: int, ratio: float, eq_ranks, rank: int, idx, counts, offsets, workspace,
                           status=None, stream=None):
    """Last step: this rank's kept positions (CSR over its own heads)."""
    _need_cuda(S, eq_ranks, idx, counts, offsets, workspace, status)
    B, n_c, nbytes = _dist_args(S, workspace)
    _check("kvz_select_dist_finish", lib().kvz_select_dist_finish(
        _ptr(S), B, n_c, int(B_total), float(ratio), _ptr(eq_ranks), int(rank), _ptr(idx), idx.numel(),
        _ptr(counts), _ptr(offsets), _ptr(workspace), nbytes, _ptr(status), _stream(stream)))


def kvz_compact_workspace_size(B: int, n_c: int) -> int:
    return lib().kvz_compact_workspace_size(B, n_c)


def kvz_compact(K, V, idx, counts, offsets, out_offsets=None, K_out=None, V_out=None, in_place: bool = False,
                out_rows: Optional[int] = None, workspace=None, status=None, stream=None):
    """Gather kept rows in key order (KVzip §2.1 pruned cache); returns (K_out, V_out).

    Out of place, the outputs are [rows, d] with head b's rows starting at
    out_offsets[b] (default offsets[b]); ``out_rows`` sizes freshly allocated
    outputs (default B*n_c, an upper bound).  In place, K and V themselves
    are returned, each head's kept rows packed to the front of its region.
    """
    _need_cuda(K, V, idx, counts, offsets, out_offsets, K_out, V_out, workspace, status)
    if K.dim() != 3 or K.shape != V.shape or K.dtype != torch.bfloat16 or V.dtype != torch.bfloat16:
        raise ValueError("K and V must be bfloat16 [B, n_c, d] of equal shape")
    B, n_c, d = K.shape
    if in_place:
        K_out, V_out = K, V
        if workspace is None:
            workspace = torch.empty(kvz_compact_workspace_size(B, n_c), dtype=torch.uint8, device=K.device)
    else:
        rows = B * n_c if out_rows is None else int(out_rows)
        if K_out is None:
            K_out = torch.empty((rows, d), dtype=K.dtype, device=K.device)
        if V_out is None:
            V_out = torch.empty((rows, d), dtype=V.dtype, device=V.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("kvz_compact", lib().kvz_compact(_ptr(K), _ptr(V), B, n_c, d, _ptr(idx), _ptr(counts), _ptr(offsets),
                                            _ptr(out_offsets), _ptr(K_out), _ptr(V_out), _ptr(workspace), ws_bytes,
                                            _ptr(status), _stream(stream)))
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
    for t in (Q, K_ctx, K_in, V):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("kvz_compress_host: Q, K_ctx, K_in and V must be contiguous bfloat16 CPU tensors")
    _need_cuda(workspace, status)
    B, G, n_in, d = Q.shape
    n_c = K_ctx.shape[1]
    if K_ctx.shape != (B, n_c, d) or V.shape != (B, n_c, d) or K_in.shape != (B, n_in, d):
        raise ValueError("kvz_compress_host: shapes must be Q [B,G,n_in,d], K_ctx/V [B,n_c,d], K_in [B,n_in,d]")
    m = _mode(mode)
    k = kvz_keep_count(B * n_c if m == GLOBAL else n_c, ratio)
    kept = k if m == GLOBAL else B * k
    if out is None:
        pin = Q.is_pinned()
        out = {"idx": torch.empty(max(kept, 1), dtype=torch.int32, pin_memory=pin),
               "counts": torch.empty(B, dtype=torch.int32, pin_memory=pin),
               "offsets": torch.empty(B + 1, dtype=torch.int64, pin_memory=pin),
               "K_out": torch.empty((max(kept, 1), d), dtype=torch.bfloat16, pin_memory=pin),
               "V_out": torch.empty((max(kept, 1), d), dtype=torch.bfloat16, pin_memory=pin)}
    if workspace is None:
        workspace = torch.empty(kvz_compress_host_workspace_size(B, G, n_c, n_in, d, ratio, m), dtype=torch.uint8,
                                device="cuda")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    st = _stream(stream)
    cst = _stream(copy_stream) if copy_stream is not None else st
    _check("kvz_compress_host", lib().kvz_compress_host(
        _ptr(Q), _ptr(K_ctx), _ptr(K_in), _ptr(V), B, G, n_c, n_in, d, float(scale), float(ratio), m,
        _ptr(out["idx"]), out["idx"].numel(), _ptr(out["counts"]), _ptr(out["offsets"]), _ptr(out["K_out"]),
        _ptr(out["V_out"]), _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status), st, cst))
    return out


def kvz_score_chunked_workspace_size(B: int, G: int, n_c: int, n_prompt: int, m: int) -> int:
    return lib().kvz_score_chunked_workspace_size(B, G, n_c, n_prompt, m)


def kvz_score_chunked(Q, Q_tail, K_ctx, K_in, K_in_tail, m: int, scale: Optional[float] = None, S=None,
                      workspace=None, status=None, stream=None):
    """Chunked importance scores (KVzip §3.4); returns S [B, n_c] fp32.

    Q [B, T, G, n_prompt+m, d] and K_in [B, T, n_prompt+m, d] hold the T full
    chunks' inputs, Q_tail / K_in_tail the shorter last chunk's (None when m
    divides n_c); K_ctx is [B, n_c, d]."""
    _need_cuda(Q, Q_tail, K_ctx, K_in, K_in_tail, S, workspace, status)
    B, n_c, d = K_ctx.shape
    T, m_last = n_c // m, n_c % m
    ref = Q if Q is not None else Q_tail
    G = ref.shape[-3]
    n_prompt = (Q.shape[-2] - m) if Q is not None else (Q_tail.shape[-2] - m_last)
    if T > 0 and (Q is None or Q.shape != (B, T, G, n_prompt + m, d) or K_in is None
                  or K_in.shape != (B, T, n_prompt + m, d)):
        raise ValueError("kvz_score_chunked: Q must be [B, T, G, n_prompt+m, d] and K_in [B, T, n_prompt+m, d]")
    if m_last > 0 and (Q_tail is None or Q_tail.shape != (B, G, n_prompt + m_last, d) or K_in_tail is None
                       or K_in_tail.shape != (B, n_prompt + m_last, d)):
        raise ValueError("kvz_score_chunked: Q_tail must be [B, G, n_prompt+m_last, d] and K_in_tail "
                         "[B, n_prompt+m_last, d]")
    if S is None:
        S = torch.empty((B, n_c), dtype=torch.float32, device=K_ctx.device)
    if workspace is None:
        workspace = torch.empty(kvz_score_chunked_workspace_size(B, G, n_c, n_prompt, m), dtype=torch.uint8,
                                device=K_ctx.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    _check("kvz_score_chunked", lib().kvz_score_chunked(
        _ptr(Q), _ptr(Q_tail), _ptr(K_ctx), _ptr(K_in), _ptr(K_in_tail), B, G, n_c, n_prompt, m, d, float(scale),
        _ptr(S), _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream)))
    return S


def kvz_head_score(S, S_head=None, status=None, stream=None):
    """Context-independent head scores (KVzip §4.2): S_head[b] = max_j S[b, j]."""
    _need_cuda(S, S_head, status)
    B, n_c = S.shape
    if S_head is None:
        S_head = torch.empty(B, dtype=torch.float32, device=S.device)
    _check("kvz_head_score", lib().kvz_head_score(_ptr(S), B, n_c, _ptr(S_head), _ptr(status), _stream(stream)))
    return S_head


def kvz_select_heads(S_head, n_c: int, ratio: float, idx=None, counts=None, offsets=None, workspace=None,
                     status=None, stream=None):
    """Head-level eviction: keep the floor(ratio*B) best heads whole; returns
    (idx, counts, offsets) in kvz_select's form, ready for kvz_compact."""
    _need_cuda(S_head, idx, counts, offsets, workspace, status)
    B = S_head.shape[0]
    k = kvz_keep_count(B, ratio)
    dev = S_head.device
    if idx is None:
        idx = torch.empty(max(1, k * n_c), dtype=torch.int32, device=dev)
    if counts is None:
        counts = torch.empty(B, dtype=torch.int32, device=dev)
    if offsets is None:
        offsets = torch.empty(B + 1, dtype=torch.int64, device=dev)
    if workspace is None:
        workspace = torch.empty(lib().kvz_select_heads_workspace_size(B), dtype=torch.uint8, device=dev)
    _check("kvz_select_heads", lib().kvz_select_heads(
        _ptr(S_head), B, n_c, float(ratio), _ptr(idx), idx.numel(), _ptr(counts), _ptr(offsets), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream)))
    return idx, counts, offsets


def kvz_decode(q, K_out, V_out, counts, offsets, n_c: int, scale: Optional[float] = None, out=None, lse2=None,
               workspace=None, status=None, stream=None):
    """One decode step of attention over the pruned cache; returns (out [B, G, d]
    fp32, lse2 [B, G] fp32).  q is bf16 [B, G, d]; K_out / V_out are the packed
    [rows, d] caches kvz_compact writes; n_c bounds every head's count."""
    _need_cuda(q, K_out, V_out, counts, offsets, out, lse2, workspace, status)
    B, G, d = q.shape
    dev = q.device
    if out is None:
        out = torch.empty((B, G, d), dtype=torch.float32, device=dev)
    if lse2 is None:
        lse2 = torch.empty((B, G), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(lib().kvz_decode_workspace_size(B, G, n_c, d), dtype=torch.uint8, device=dev)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    _check("kvz_decode", lib().kvz_decode(
        _ptr(q), _ptr(K_out), _ptr(V_out), K_out.shape[0], _ptr(counts), _ptr(offsets), B, G, n_c, d, float(scale),
        _ptr(out), _ptr(lse2), _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)))
    return out, lse2


def kvz_select_protected(S, ratio: float, mode="per_head", n_protect: int = 0, idx=None, counts=None, offsets=None,
                         workspace=None, status=None, stream=None):
    """kvz_select with the first n_protect positions of every head always
    kept (KVzip §4.1 system prompt); the ratio applies to the rest."""
    _need_cuda(S, idx, counts, offsets, workspace, status)
    B, n_c = S.shape
    m = _mode(mode)
    free = n_c - n_protect
    k = (B * n_protect + kvz_keep_count(B * free, ratio)) if m == GLOBAL else (n_protect + kvz_keep_count(free, ratio))
    cap = k if m == GLOBAL else B * k
    dev = S.device
    if idx is None:
        idx = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
    if counts is None:
        counts = torch.empty(B, dtype=torch.int32, device=dev)
    if offsets is None:
        offsets = torch.empty(B + 1, dtype=torch.int64, device=dev)
    if workspace is None:
        workspace = torch.empty(kvz_select_workspace_size(B, n_c, m), dtype=torch.uint8, device=dev)
    _check("kvz_select_protected", lib().kvz_select_protected(
        _ptr(S), B, n_c, float(ratio), m, int(n_protect), _ptr(idx), idx.numel(), _ptr(counts), _ptr(offsets),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream)))
    return idx, counts, offsets


def kvz_compact_int8(K, V, idx, counts, offsets, out_offsets=None, out_rows: Optional[int] = None, Kq=None, Vq=None,
                     K_scale=None, V_scale=None, status=None, stream=None):
    """Out-of-place compaction into int8 codes with one fp32 scale per row
    (KVzip §4.2 KV quantisation); returns (Kq, K_scale, Vq, V_scale)."""
    _need_cuda(K, V, idx, counts, offsets, out_offsets, Kq, Vq, K_scale, V_scale, status)
    B, n_c, d = K.shape
    rows = B * n_c if out_rows is None else int(out_rows)
    dev = K.device
    Kq = torch.empty((rows, d), dtype=torch.int8, device=dev) if Kq is None else Kq
    Vq = torch.empty((rows, d), dtype=torch.int8, device=dev) if Vq is None else Vq
    K_scale = torch.empty(rows, dtype=torch.float32, device=dev) if K_scale is None else K_scale
    V_scale = torch.empty(rows, dtype=torch.float32, device=dev) if V_scale is None else V_scale
    _check("kvz_compact_int8", lib().kvz_compact_int8(
        _ptr(K), _ptr(V), B, n_c, d, _ptr(idx), _ptr(counts), _ptr(offsets), _ptr(out_offsets), _ptr(Kq), _ptr(Vq),
        _ptr(K_scale), _ptr(V_scale), _ptr(status), _stream(stream)))
    return Kq, K_scale, Vq, V_scale
