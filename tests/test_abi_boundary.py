"""Argument validation of the C ABI: every rejected call returns its status
before anything is launched.  Runs on the GPU with real, correctly sized
buffers (so a validation bug could not reach a kernel with a bad pointer)
and on the CPU with placeholder addresses (nothing is launched there)."""
import ctypes

import pytest
import torch

import query_agnostic_kv_kvz_b200 as kvz

OK, INVALID, UNSUPPORTED, ALIGN, WS = 0, 1, 2, 3, 4


class Bufs:
    """Device buffers when CUDA is present, else fake 256-aligned addresses."""

    def __init__(self):
        self.cuda = torch.cuda.is_available()
        self.keep = []
        self.fake = 1 << 20

    def get(self, nbytes):
        if self.cuda:
            t = torch.zeros(max(16, nbytes), dtype=torch.uint8, device="cuda")
            self.keep.append(t)
            return t.data_ptr()
        self.fake += ((nbytes + 255) // 256 + 1) * 256
        return self.fake


@pytest.fixture(scope="module")
def lib():
    from query_agnostic_kv_kvz_b200 import build
    build.build()
    return kvz.lib()


def vp(x):
    return ctypes.c_void_p(x)


def _score(lib, bufs, B=1, G=1, n_c=128, n_in=128, d=128, scale=0.1, row_chunk=0, ws_bytes=None,
           shift=0, ws_ptr=True):
    Q = bufs.get(B * G * n_in * d * 2) + shift
    Kc = bufs.get(B * n_c * d * 2)
    Ki = bufs.get(B * n_in * d * 2)
    S = bufs.get(B * n_c * 4)
    need = lib.kvz_score_workspace_size(B, G, n_in, row_chunk if row_chunk % 256 == 0 else 0)
    ws = bufs.get(need) if ws_ptr else 0
    return lib.kvz_score(vp(Q), vp(Kc), vp(Ki), B, G, n_c, n_in, d, scale, row_chunk, vp(S), vp(ws),
                         need if ws_bytes is None else ws_bytes, None, None)


def test_score_rejections(lib):
    b = Bufs()
    assert _score(lib, b, d=96) == UNSUPPORTED
    assert _score(lib, b, d=256) == UNSUPPORTED
    assert _score(lib, b, scale=0.0) == INVALID
    assert _score(lib, b, scale=float("nan")) == INVALID
    assert _score(lib, b, scale=float("inf")) == INVALID
    assert _score(lib, b, G=0) == INVALID
    assert _score(lib, b, n_c=0) == INVALID
    assert _score(lib, b, row_chunk=100) == INVALID
    assert _score(lib, b, shift=2) == ALIGN
    assert _score(lib, b, ws_bytes=16) == WS
    assert _score(lib, b, ws_ptr=False) == WS
    assert lib.kvz_score(None, None, None, 1, 1, 8, 8, 128, 0.1, 0, None, None, 0, None, None) == INVALID


def test_pass_rejections(lib):
    b = Bufs()
    Q, Kc, Ki = b.get(4 * 512 * 128 * 2), b.get(512 * 128 * 2), b.get(512 * 128 * 2)
    lse = b.get(4 * 512 * 4)
    S = b.get(512 * 4)
    ws = b.get(lib.kvz_score_lse2_workspace_size())

    def lse2(i0=0, i1=512, ld=512, shift=0, ws_bytes=None, ws_ptr=True):
        return lib.kvz_score_lse2(vp(Q), vp(Kc), vp(Ki), 1, 4, 512, 512, 128, 0.1, i0, i1, vp(lse), ld,
                                  vp(ws + shift) if ws_ptr else None,
                                  lib.kvz_score_lse2_workspace_size() if ws_bytes is None else ws_bytes, None, None)
    # i_begin not a multiple of 256, range outside n_in, ld too small
    assert lse2(i0=100) == INVALID
    assert lse2(i1=513) == INVALID
    assert lse2(ld=256) == INVALID
    assert lse2(ld=510) == ALIGN
    # the optional workspace: too small, misaligned
    assert lse2(ws_bytes=1024) == WS
    assert lse2(shift=8) == ALIGN
    assert lib.kvz_score_lse2_workspace_size() >= 256 * 256 * 8
    assert lib.kvz_score_colmax(vp(Q), vp(Kc), 1, 4, 512, 512, 128, 0.1, 256, 128, vp(lse), 512, vp(S), 0, None,
                                None) == INVALID
    assert lib.kvz_score_colmax(vp(Q), vp(Kc), 1, 4, 512, 512, 128, 0.1, 0, 512, None, 512, vp(S), 0, None,
                                None) == INVALID


def test_select_rejections(lib):
    b = Bufs()
    B, n_c = 4, 1000
    S = b.get(B * n_c * 4)
    idx, cnt, off = b.get(B * n_c * 4), b.get(B * 4), b.get((B + 1) * 8)
    ws_n = lib.kvz_select_workspace_size(B, n_c, 0)
    ws = b.get(ws_n)

    def call(ratio=0.3, mode=0, cap=B * n_c, wsb=ws_n, s_shift=0, Bx=B):
        return lib.kvz_select(vp(S + s_shift), Bx, n_c, ratio, mode, vp(idx), cap, vp(cnt), vp(off), vp(ws), wsb,
                              None, None)

    assert call(ratio=1.5) == INVALID
    assert call(ratio=-0.1) == INVALID
    assert call(ratio=float("nan")) == INVALID
    assert call(mode=3) == INVALID
    assert call(cap=B * 300 - 1) == INVALID          # per head: 4 * floor(0.3*1000) = 1200 needed
    assert call(wsb=16) == WS
    assert call(s_shift=2) == ALIGN
    assert call(Bx=70000) == INVALID


def test_compact_rejections(lib):
    b = Bufs()
    B, n_c, d = 2, 256, 128
    K, V = b.get(B * n_c * d * 2), b.get(B * n_c * d * 2)
    Ko, Vo = b.get(B * n_c * d * 2), b.get(B * n_c * d * 2)
    idx, cnt, off = b.get(B * n_c * 4), b.get(B * 4), b.get((B + 1) * 8)
    outo = b.get((B + 1) * 8)

    ws = b.get(lib.kvz_compact_workspace_size(B, n_c))

    def call(K_=K, V_=V, Ko_=Ko, Vo_=Vo, d_=d, oo=None, ws_=ws, wsb=None):
        wsb = lib.kvz_compact_workspace_size(B, n_c) if wsb is None else wsb
        return lib.kvz_compact(vp(K_), vp(V_), B, n_c, d_, vp(idx), vp(cnt), vp(off), vp(oo) if oo else None,
                               vp(Ko_), vp(Vo_), vp(ws_) if ws_ else None, wsb, None, None)

    assert call(d_=96) == UNSUPPORTED
    assert call(Ko_=K) == INVALID                    # K in place, V not
    assert call(Ko_=K, Vo_=V, oo=outo) == INVALID    # in place takes no output offsets
    assert call(V_=K) == INVALID                     # K and V are the same buffer
    assert call(Ko_=K + 4096) == INVALID             # output starts inside an input
    assert call(Ko_=Ko + 8) == ALIGN
    assert call(Ko_=K, Vo_=V, ws_=0) == WS           # in place needs the progress counters
    assert call(Ko_=K, Vo_=V, wsb=8) == WS
    assert lib.kvz_compact(vp(K), vp(V), B, n_c, d, None, vp(cnt), vp(off), None, vp(Ko), vp(Vo), None, 0,
                           None, None) == INVALID


def test_compress_host_rejections(lib):
    b = Bufs()
    B, G, n_c, n_in, d = 2, 2, 1000, 1032, 128
    hQ, hK, hKi, hV = (ctypes.create_string_buffer(16) for _ in range(4))   # never read: every call is rejected
    hidx, hcnt, hoff, hko, hvo = (ctypes.create_string_buffer(16) for _ in range(5))
    need = lib.kvz_compress_host_workspace_size(B, G, n_c, n_in, d, 0.3, 0)
    assert need > 2 * (B * G * n_in + 2 * B * n_c + B * n_in) * d     # holds the device copies of the inputs
    ws = b.get(need)
    kept = B * 300

    def call(d_=d, scale=0.1, ratio=0.3, mode=0, cap=kept, wsb=need, ws_=ws, q=hQ):
        return lib.kvz_compress_host(q, hK, hKi, hV, B, G, n_c, n_in, d_, scale, ratio, mode, hidx, cap, hcnt, hoff,
                                     hko, hvo, vp(ws_) if ws_ else None, wsb, None, None, None)

    assert call(d_=96) == UNSUPPORTED
    assert call(scale=0.0) == INVALID
    assert call(ratio=1.5) == INVALID
    assert call(mode=2) == INVALID
    assert call(cap=kept - 1) == INVALID
    assert call(q=None) == INVALID
    assert call(wsb=need - 1) == WS
    assert call(ws_=0) == WS
    assert lib.kvz_compress_host_workspace_size(B, G, n_c, n_in, 96, 0.3, 0) == 0


def test_score_chunked_rejections(lib):
    b = Bufs()
    B, G, n_c, n_prompt, m, d = 2, 4, 700, 16, 256, 128
    T, ml = n_c // m, n_c % m
    Q, Qt = b.get(B * T * G * (n_prompt + m) * d * 2), b.get(B * G * (n_prompt + ml) * d * 2)
    Kc = b.get(B * n_c * d * 2)
    Ki, Kit = b.get(B * T * (n_prompt + m) * d * 2), b.get(B * (n_prompt + ml) * d * 2)
    S = b.get(B * n_c * 4)
    need = lib.kvz_score_chunked_workspace_size(B, G, n_c, n_prompt, m)
    # the full chunks' rows, padded to 256, dominate; plus pass 1's split-tail scratch
    assert need == B * T * G * 512 * 4 + lib.kvz_score_lse2_workspace_size()
    ws = b.get(need)

    def call(q=Q, qt=Qt, d_=d, m_=m, wsb=need, scale=0.1):
        return lib.kvz_score_chunked(vp(q) if q else None, vp(qt) if qt else None, vp(Kc), vp(Ki), vp(Kit), B, G,
                                     n_c, n_prompt, m_, d_, scale, vp(S), vp(ws), wsb, None, None)

    assert call(d_=96) == UNSUPPORTED
    assert call(m_=0) == INVALID
    assert call(q=0) == INVALID                  # full chunks exist but no Q
    assert call(qt=0) == INVALID                 # a tail exists but no Q_tail
    assert call(scale=float("nan")) == INVALID
    assert call(wsb=need - 1) == WS
    assert call(q=Q + 8) == ALIGN
    assert lib.kvz_score_chunked_workspace_size(B, G, n_c, n_prompt, 0) == 0


def test_head_rejections(lib):
    b = Bufs()
    B, n_c = 8, 100
    S, H = b.get(B * n_c * 4), b.get(B * 4)
    idx, cnt, off = b.get(4 * n_c * 4), b.get(B * 4), b.get((B + 1) * 8)
    need = lib.kvz_select_heads_workspace_size(B)
    ws = b.get(need)
    assert lib.kvz_head_score(vp(S), 0, n_c, vp(H), None, None) == INVALID
    assert lib.kvz_head_score(vp(S + 2), B, n_c, vp(H), None, None) == ALIGN
    assert lib.kvz_head_score(None, B, n_c, vp(H), None, None) == INVALID

    def sel(ratio=0.5, cap=4 * n_c, wsb=need):
        return lib.kvz_select_heads(vp(H), B, n_c, ratio, vp(idx), cap, vp(cnt), vp(off), vp(ws), wsb, None, None)

    assert sel(ratio=1.2) == INVALID
    assert sel(cap=4 * n_c - 1) == INVALID         # 4 heads of 100 rows each
    assert sel(wsb=need - 1) == WS
    assert lib.kvz_select_heads_workspace_size(70000) == 0


def test_decode_rejections(lib):
    b = Bufs()
    B, G, n_c, d = 2, 4, 500, 128
    q, K, V = b.get(B * G * d * 2), b.get(B * n_c * d * 2), b.get(B * n_c * d * 2)
    cnt, off = b.get(B * 4), b.get((B + 1) * 8)
    out, lse = b.get(B * G * d * 4), b.get(B * G * 4)
    need = lib.kvz_decode_workspace_size(B, G, n_c, d)
    assert need > 0
    ws = b.get(need)

    def call(G_=G, d_=d, wsb=need, qq=q, scale=0.1):
        return lib.kvz_decode(vp(qq), vp(K), vp(V), B * n_c, vp(cnt), vp(off), B, G_, n_c, d_, scale, vp(out),
                              vp(lse), vp(ws), wsb, None, None)

    assert call(d_=96) == UNSUPPORTED
    assert call(G_=9) == UNSUPPORTED
    assert call(scale=-1.0) == INVALID
    assert call(wsb=need - 1) == WS
    assert call(qq=q + 2) == ALIGN
    assert lib.kvz_decode_workspace_size(B, 9, n_c, d) == 0


def test_protect_and_int8_rejections(lib):
    b = Bufs()
    B, n_c, d = 2, 256, 128
    S = b.get(B * n_c * 4)
    idx, cnt, off = b.get(B * n_c * 4), b.get(B * 4), b.get((B + 1) * 8)
    wsn = lib.kvz_select_workspace_size(B, n_c, 0)
    ws = b.get(wsn)
    sel = lambda p, cap=B * n_c: lib.kvz_select_protected(vp(S), B, n_c, 0.3, 0, p, vp(idx), cap, vp(cnt), vp(off),
                                                        vp(ws), wsn, None, None)
    assert sel(-1) == INVALID
    assert sel(n_c + 1) == INVALID
    assert sel(10, cap=B * (10 + 73) - 1) == INVALID      # per head: 10 + floor(0.3 * 246) = 83
    K, V = b.get(B * n_c * d * 2), b.get(B * n_c * d * 2)
    Kq, Vq, Ks, Vs = b.get(B * n_c * d), b.get(B * n_c * d), b.get(B * n_c * 4), b.get(B * n_c * 4)
    q8 = lambda d_=d, kq=Kq: lib.kvz_compact_int8(vp(K), vp(V), B, n_c, d_, vp(idx), vp(cnt), vp(off), None, vp(kq),
                                                 vp(Vq), vp(Ks), vp(Vs), None, None)
    assert q8(d_=96) == UNSUPPORTED
    assert q8(kq=Kq + 8) == ALIGN


def test_select_dist_rejections(lib):
    b = Bufs()
    B, n_c, B_total = 3, 1000, 8
    S = b.get(B * n_c * 4)
    hist, eq, eqr = b.get(2048 * 4), b.get(16), b.get(8 * 8)
    idx, cnt, off = b.get(B * n_c * 4), b.get(B * 4), b.get((B + 1) * 8)
    ws_n = lib.kvz_select_dist_workspace_size(B, n_c)
    assert ws_n > 0 and lib.kvz_select_dist_workspace_size(0, n_c) == 0
    ws = b.get(ws_n)

    def begin(Bt=B_total, ratio=0.3, h=hist, wsb=ws_n, s=S):
        return lib.kvz_select_dist_begin(vp(s), B, n_c, Bt, ratio, vp(h) if h else None, vp(ws), wsb, None, None)

    def step(p=0, h=hist, e=eq, wsb=ws_n):
        return lib.kvz_select_dist_step(vp(S), B, n_c, p, vp(h) if h else None, vp(e) if e else None, vp(ws), wsb,
                                        None, None)

    def finish(Bt=B_total, ratio=0.3, er=eqr, rank=1, cap=B * n_c, wsb=ws_n):
        return lib.kvz_select_dist_finish(vp(S), B, n_c, Bt, ratio, vp(er) if er else None, rank, vp(idx), cap,
                                          vp(cnt), vp(off), vp(ws), wsb, None, None)

    assert begin(Bt=B - 1) == INVALID                 # fewer heads in all than on this rank
    assert begin(ratio=1.01) == INVALID
    assert begin(h=None) == INVALID
    assert begin(h=hist + 4) == ALIGN
    assert begin(wsb=ws_n - 1) == WS
    assert begin(s=S + 2) == ALIGN
    assert begin(Bt=(1 << 32) // n_c + 1) == INVALID  # 32-bit histogram bins
    assert step(p=3) == INVALID
    assert step(p=-1) == INVALID
    assert step(p=2, e=None) == INVALID               # the last step writes the equal-key total
    assert step(h=None) == INVALID
    assert step(e=eq + 4) == ALIGN
    assert finish(er=None) == INVALID
    assert finish(rank=-1) == INVALID
    assert finish(cap=int(0.3 * B_total * n_c) - 1) == INVALID   # min(k, B*n_c) = 2400 slots needed
    assert finish(er=eqr + 4) == ALIGN
    assert finish(wsb=0) == WS
