"""bench.py's work accounting, the numerators of every throughput and
roofline figure, against counts taken from the definition by brute force on
small shapes: visible (row, key) pairs under the causal mask, context-key
pairs of pass 2, kept rows, and the compaction's algorithmic bytes."""
import dataclasses
import importlib.util
import math
import os

import pytest

from query_agnostic_kv_kvz_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def brute(w):
    pairs1 = pairs2 = kept = 0
    for n_c in w.n_c:
        if w.chunk:
            blocks = [(min(w.chunk, n_c - c0), w.n_prompt + min(w.chunk, n_c - c0)) for c0 in range(0, n_c, w.chunk)]
        else:
            blocks = [(n_c, w.n_prompt + n_c)]
        for nk, ni in blocks:
            for i in range(ni):                      # input row i sees nk context keys + input keys 0..i
                pairs1 += w.B * w.G * (nk + i + 1)
                pairs2 += w.B * w.G * nk
        free = n_c - w.n_protect
        if w.mode == "global":
            kept += w.B * w.n_protect + math.floor(w.ratio * w.B * free)
        elif w.mode == "heads":
            kept += math.floor(w.ratio * w.B) * n_c
        else:
            kept += w.B * (w.n_protect + math.floor(w.ratio * free))
    return pairs1, pairs2, kept


@pytest.mark.parametrize("name,L,n_c", [("tiny", 1, None), ("llama8b_layer", 1, (300,)), ("qwen14b_128k", 2, (257,)),
                                        ("stress_ragged", 1, (10, 33, 65)), ("llama8b_170k_chunked", 1, (1000,)),
                                        ("llama8b_stack_int8", 2, (200,)), ("llama8b_stack_heads", 3, (50,))])
def test_work_numbers_match_brute_force(bench, name, L, n_c):
    w = synth.WORKLOADS[name]
    w = dataclasses.replace(w, L=L, **({"n_c": n_c} if n_c else {}))
    if w.chunk:
        w = dataclasses.replace(w, chunk=128)
    nums = bench.workload_numbers(w)
    p1, p2, kept = brute(w)
    assert nums["pairs_per_step"] == w.B * sum(w.n_c)
    assert nums["flops_pass1"] == 2 * w.d * p1
    assert nums["flops_pass2"] == 2 * w.d * p2
    assert nums["kept"] == kept
    row = w.d * 2
    if w.quant:   # bf16 K and V read, int8 K and V and two fp32 scales written, idx read
        assert nums["compact_bytes"] == kept * (2 * row + 2 * w.d + 8) + 4 * kept
    else:         # K and V rows read and written, idx read
        assert nums["compact_bytes"] == kept * 4 * row + 4 * kept


def test_headline_flops_of_the_128k_config(bench):
    # one QK^T over the visible pairs of 48 x 8 heads, G=5, n_c=131072,
    # n_in=131104: 2 * 128 * 384 * 5 * (n_in * n_c + n_in (n_in + 1) / 2)
    nums = bench.workload_numbers(synth.WORKLOADS["qwen14b_128k"])
    n_c, n_in = 131072, 131104
    assert nums["flops_pass1"] == 2 * 128 * 384 * 5 * (n_in * n_c + n_in * (n_in + 1) // 2)
    assert abs(nums["flops_pass1"] / 1.267e16 - 1) < 2e-3
    assert nums["compact_bytes"] == 384 * 32768 * (4 * 256 + 4)
