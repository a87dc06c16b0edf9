"""The Python binding rejects malformed tensors before anything reaches the
C ABI, which trusts the buffer sizes it is given.  Runs on the CPU: the
library is replaced by a stand-in whose size helpers answer and whose
compute entry points fail the test if they are ever called."""
import math

import pytest
import torch

import query_agnostic_kv_kvz_b200 as kvz

bf16, f32, i32, i64, u8, i8 = torch.bfloat16, torch.float32, torch.int32, torch.int64, torch.uint8, torch.int8


class _NoLaunchLib:
    """Size helpers answer; every other entry point is a test failure."""

    def __getattr__(self, name):
        if name.endswith("_workspace_size"):
            return lambda *a: 1 << 16
        if name == "kvz_keep_count":
            return lambda n, r: int(math.floor(r * n))
        def launched(*a):
            raise AssertionError("%s reached the C ABI with a malformed argument" % name)
        return launched


@pytest.fixture(autouse=True)
def _no_launch(monkeypatch):
    monkeypatch.setattr(kvz, "lib", lambda: _NoLaunchLib())


def z(shape, dtype):
    return torch.zeros(shape, dtype=dtype)


B, G, n_in, n_c, d = 2, 3, 40, 50, 64
Q, Kc, Ki = z((B, G, n_in, d), bf16), z((B, n_c, d), bf16), z((B, n_in, d), bf16)
S = z((B, n_c), f32)
cnt, off = z(B, i32), z(B + 1, i64)
idx = z(B * 15, i32)
rows = B * 15

CASES = {
    # scoring
    "score: Q not bf16": lambda: kvz.kvz_score(Q.float(), Kc, Ki),
    "score: K_in rows": lambda: kvz.kvz_score(Q, Kc, z((B, n_in - 1, d), bf16)),
    "score: K_ctx heads": lambda: kvz.kvz_score(Q, z((B + 1, n_c, d), bf16), Ki),
    "score: S shape": lambda: kvz.kvz_score(Q, Kc, Ki, S=z((B, n_c - 1), f32)),
    "score: S dtype": lambda: kvz.kvz_score(Q, Kc, Ki, S=z((B, n_c), torch.float64)),
    "score: workspace dtype": lambda: kvz.kvz_score(Q, Kc, Ki, workspace=z(100, f32)),
    "score: status dtype": lambda: kvz.kvz_score(Q, Kc, Ki, status=z(1, i64)),
    "score: non-contiguous Q": lambda: kvz.kvz_score(z((B, G, d, n_in), bf16).transpose(2, 3), Kc, Ki),
    "score: CPU tensors": lambda: kvz.kvz_score(Q, Kc, Ki),
    "noalloc: S shape": lambda: kvz.kvz_score_noalloc(Q, Kc, Ki, S=z((B * n_c,), f32)),
    "noalloc: CPU tensors": lambda: kvz.kvz_score_noalloc(Q, Kc, Ki),
    "lse2: ld too small": lambda: kvz.kvz_score_lse2(Q, Kc, Ki, lse2=z((B, G, 128), f32)),
    "lse2: i_begin unaligned": lambda: kvz.kvz_score_lse2(Q, Kc, Ki, i_begin=8),
    "colmax: lse2 heads": lambda: kvz.kvz_score_colmax(Q, Kc, z((B + 1, G, 256), f32)),
    "colmax: accumulate without S": lambda: kvz.kvz_score_colmax(Q, Kc, z((B, G, 256), f32), accumulate=True),
    "chunked: K_in_tail shape": lambda: kvz.kvz_score_chunked(None, z((B, G, 10 + 5, d), bf16), z((B, 5, d), bf16),
                                                           None, z((B, 16, d), bf16), 8),
    # selection
    "select: S rank": lambda: kvz.kvz_select(z(n_c, f32), 0.3),
    "select: idx short": lambda: kvz.kvz_select(S, 0.3, idx=z(B * 15 - 1, i32)),
    "select: counts dtype": lambda: kvz.kvz_select(S, 0.3, counts=z(B, i64)),
    "select: offsets short": lambda: kvz.kvz_select(S, 0.3, offsets=z(B, i64)),
    "select: ratio": lambda: kvz.kvz_select(S, 1.5),
    "protected: n_protect > n_c": lambda: kvz.kvz_select_protected(S, 0.3, n_protect=n_c + 1),
    "protected: idx short": lambda: kvz.kvz_select_protected(S, 0.3, "global", 4, idx=z(8 + 27 - 1, i32)),
    "head_score: S dtype": lambda: kvz.kvz_head_score(S.double()),
    "head_score: S_head short": lambda: kvz.kvz_head_score(S, S_head=z(B - 1, f32)),
    "select_heads: S_head rank": lambda: kvz.kvz_select_heads(z((B, 1), f32), n_c, 0.5),
    "select_heads: idx short": lambda: kvz.kvz_select_heads(z(4, f32), n_c, 0.5, idx=z(2 * n_c - 1, i32)),
    "select_heads: offsets dtype": lambda: kvz.kvz_select_heads(z(4, f32), n_c, 0.5, offsets=z(5, i32)),
    "dist_begin: hist short": lambda: kvz.kvz_select_dist_begin(S, B, 0.3, z(2047, i32), z(64, u8)),
    "dist_step: eq_total dtype": lambda: kvz.kvz_select_dist_step(S, 2, z(2048, i32), z(1, i32), z(64, u8)),
    "dist_finish: eq_ranks short": lambda: kvz.kvz_select_dist_finish(S, B, 0.3, z(1, i64), 1, idx, cnt, off,
                                                                     z(64, u8)),
    # compaction
    "compact: idx dtype": lambda: kvz.kvz_compact(Kc, Kc.clone(), idx.long(), cnt, off),
    "compact: K/V shapes": lambda: kvz.kvz_compact(Kc, z((B, n_c, d + 8), bf16), idx, cnt, off),
    "compact: K_out rows": lambda: kvz.kvz_compact(Kc, Kc.clone(), idx, cnt, off, K_out=z((rows - 1, d), bf16)),
    "compact: V_out width": lambda: kvz.kvz_compact(Kc, Kc.clone(), idx, cnt, off, V_out=z((rows, d // 2), bf16)),
    "compact: out_rows": lambda: kvz.kvz_compact(Kc, Kc.clone(), idx, cnt, off, out_rows=rows - 1),
    "compact: counts short": lambda: kvz.kvz_compact(Kc, Kc.clone(), idx, z(B - 1, i32), off),
    "compact: in place with K_out": lambda: kvz.kvz_compact(Kc, Kc.clone(), idx, cnt, off, in_place=True,
                                                            K_out=Kc),
    "compact: out_offsets short": lambda: kvz.kvz_compact(Kc, Kc.clone(), idx, cnt, off, out_offsets=z(B - 1, i64)),
    "int8: Kq dtype": lambda: kvz.kvz_compact_int8(Kc, Kc.clone(), idx, cnt, off, Kq=z((rows, d), u8)),
    "int8: Vq rows": lambda: kvz.kvz_compact_int8(Kc, Kc.clone(), idx, cnt, off, Vq=z((rows - 1, d), i8)),
    "int8: K_scale short": lambda: kvz.kvz_compact_int8(Kc, Kc.clone(), idx, cnt, off, Kq=z((rows, d), i8),
                                                        K_scale=z(rows - 1, f32)),
    "int8: V_scale dtype": lambda: kvz.kvz_compact_int8(Kc, Kc.clone(), idx, cnt, off, V_scale=z(B * n_c, i32)),
    "int8: offsets dtype": lambda: kvz.kvz_compact_int8(Kc, Kc.clone(), idx, cnt, off.int()),
    # decode
    "decode: q dtype": lambda: kvz.kvz_decode(z((B, G, d), f32), z((rows, d), bf16), z((rows, d), bf16), cnt, off,
                                              n_c),
    "decode: K_out width": lambda: kvz.kvz_decode(z((B, G, d), bf16), z((rows, d + 8), bf16),
                                                  z((rows, d + 8), bf16), cnt, off, n_c),
    "decode: K/V rows differ": lambda: kvz.kvz_decode(z((B, G, d), bf16), z((rows, d), bf16),
                                                      z((rows - 1, d), bf16), cnt, off, n_c),
    "decode: counts dtype": lambda: kvz.kvz_decode(z((B, G, d), bf16), z((rows, d), bf16), z((rows, d), bf16),
                                                   cnt.long(), off, n_c),
    "decode: out shape": lambda: kvz.kvz_decode(z((B, G, d), bf16), z((rows, d), bf16), z((rows, d), bf16), cnt,
                                                off, n_c, out=z((B, G, d), bf16)),
    "decode: lse2 shape": lambda: kvz.kvz_decode(z((B, G, d), bf16), z((rows, d), bf16), z((rows, d), bf16), cnt,
                                                 off, n_c, lse2=z((B * G,), f32)),
    "decode: CPU tensors": lambda: kvz.kvz_decode(z((B, G, d), bf16), z((rows, d), bf16), z((rows, d), bf16), cnt,
                                                  off, n_c),
    # host path
    "host: Q rank": lambda: kvz.kvz_compress_host(Q[0], Kc, Ki, Kc.clone(), 0.3),
    "host: out K_out rows": lambda: kvz.kvz_compress_host(
        Q, Kc, Ki, Kc.clone(), 0.3,
        out={"idx": z(rows, i32), "counts": cnt, "offsets": off, "K_out": z((rows - 1, d), bf16),
             "V_out": z((rows, d), bf16)}),
    "host: out counts dtype": lambda: kvz.kvz_compress_host(
        Q, Kc, Ki, Kc.clone(), 0.3,
        out={"idx": z(rows, i32), "counts": cnt.long(), "offsets": off, "K_out": z((rows, d), bf16),
             "V_out": z((rows, d), bf16)}),
}


# the message each case must raise: the intended check fired, not a later one
EXPECT = {
    'chunked: K_in_tail shape': 'K_in_tail must have shape',
    'colmax: accumulate without S': 'accumulate',
    'colmax: lse2 heads': 'lse2 must be [B, G, ld]',
    'compact: K/V shapes': 'K and V must be',
    'compact: K_out rows': 'K_out must be [rows >= ',
    'compact: V_out width': 'V_out must be [rows >= ',
    'compact: counts short': 'counts holds',
    'compact: idx dtype': 'idx must be torch.int32',
    'compact: in place with K_out': 'in place takes no',
    'compact: out_offsets short': 'out_offsets holds',
    'compact: out_rows': 'out_rows must be',
    'decode: CPU tensors': 'CUDA device',
    'decode: K/V rows differ': 'equal shape',
    'decode: K_out width': 'K_out must be [rows >= ',
    'decode: counts dtype': 'counts must be torch.int32',
    'decode: lse2 shape': 'lse2 must have shape',
    'decode: out shape': 'out must be torch.float32',
    'decode: q dtype': 'q must be torch.bfloat16',
    'dist_begin: hist short': 'hist holds',
    'dist_finish: eq_ranks short': 'eq_ranks holds',
    'dist_step: eq_total dtype': 'eq_total must be',
    'head_score: S dtype': 'S must be torch.float32',
    'head_score: S_head short': 'S_head holds',
    'host: Q rank': 'Q must be [B, G, n_in, d]',
    'host: out K_out rows': "out['K_out'] must be",
    'host: out counts dtype': "out['counts'] must be torch.int32",
    'int8: K_scale short': 'K_scale holds',
    'int8: Kq dtype': 'Kq must be torch.int8',
    'int8: V_scale dtype': 'V_scale must be torch.float32',
    'int8: Vq rows': 'Vq must be [rows >= ',
    'int8: offsets dtype': 'offsets must be torch.int64',
    'lse2: i_begin unaligned': 'i_begin % 256',
    'lse2: ld too small': 'ld must be',
    'noalloc: CPU tensors': 'CUDA device',
    'noalloc: S shape': 'S must have shape',
    'protected: idx short': 'idx holds',
    'protected: n_protect > n_c': 'n_protect',
    'score: CPU tensors': 'CUDA device',
    'score: K_ctx heads': 'K_ctx must be',
    'score: K_in rows': 'K_in must have shape',
    'score: Q not bf16': 'Q must be torch.bfloat16',
    'score: S dtype': 'S must be torch.float32',
    'score: S shape': 'S must have shape',
    'score: non-contiguous Q': 'Q must be contiguous',
    'score: status dtype': 'status must be torch.int32',
    'score: workspace dtype': 'workspace must be torch.uint8',
    'select: S rank': 'S must have 2 dimensions',
    'select: counts dtype': 'counts must be',
    'select: idx short': 'idx holds',
    'select: offsets short': 'offsets holds',
    'select: ratio': 'ratio must lie',
    'select_heads: S_head rank': 'S_head must have 1',
    'select_heads: idx short': 'idx holds',
    'select_heads: offsets dtype': 'offsets must be torch.int64',
}


def test_every_case_names_its_check():
    assert sorted(EXPECT) == sorted(CASES)


@pytest.mark.parametrize("case", sorted(CASES))
def test_malformed_call_raises_before_the_c_abi(case):
    with pytest.raises(ValueError) as err:
        CASES[case]()
    assert EXPECT[case] in str(err.value), str(err.value)
