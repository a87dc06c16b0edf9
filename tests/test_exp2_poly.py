"""The FMA-pipe 2^x used by score pass 1, emulated operation by operation in
float32 (coefficients read from the CUDA header), against exact 2^x."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "query_agnostic_kv_kvz_b200", "csrc", "kvz_sm100.cuh")


def coefficients():
    body = open(HDR).read().split("exp2_poly2(float2 x)")[1].split("return make_float2")[0]
    lits = re.findall(r"(0x1\.[0-9a-f]+p-?\d+)f", body)
    # fma order in the source: c4 (first operand), c3, c2, c1, c0, each written twice
    vals = [float.fromhex(s) for s in lits[::2]]
    assert len(vals) == 5
    c4, c3, c2, c1, c0 = vals
    return [np.float32(c) for c in (c0, c1, c2, c3, c4)]


def f32_fma(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def emulate(x):
    c0, c1, c2, c3, c4 = coefficients()
    shift = np.float32(12582912.0)
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + shift).astype(np.float32)
    n = (t - shift).astype(np.float32)
    f = f32_fma(n, np.float32(-1.0) * np.ones_like(n), x)
    p = f32_fma(np.full_like(f, c4), f, np.full_like(f, c3))
    p = f32_fma(p, f, np.full_like(f, c2))
    p = f32_fma(p, f, np.full_like(f, c1))
    p = f32_fma(p, f, np.full_like(f, c0))
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_reduction_is_exact_and_error_bounded():
    x = np.concatenate([np.linspace(-125.0, 8.0, 4_000_001, dtype=np.float32),
                        np.arange(-125, 9, dtype=np.float32),                 # integers
                        np.arange(-125, 8, dtype=np.float32) + np.float32(0.5)])  # ties
    y = emulate(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 3e-6, rel.max()


def test_masked_inputs_are_negligible():
    y = emulate(np.array([-np.inf, -1e30, -200.0], np.float32))
    assert np.all(y > 0) and np.all(y <= 2.0 ** -124)


def test_fit_script_reproduces_header():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "fit", os.path.join(ROOT, "query_agnostic_kv_kvz_b200", "csrc", "fit_exp2_poly.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c32, _, rel32 = fit.report(4)
    assert rel32 < 3e-6
    np.testing.assert_array_equal(np.array(coefficients(), np.float32), c32)
