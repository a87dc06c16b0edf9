"""Fit the polynomial that kvz_sm100.cuh uses for 2^f, f in [-1/2, 1/2].

The score kernels evaluate part of their exp2 work on the FMA pipe.  They
use a range reduction x = n + f with n = round(x) (obtained by adding and
subtracting 1.5 * 2^23) and 2^x = 2^n * p(f), where 2^n is added directly to
the exponent field.  p is a degree-DEG polynomial chosen to minimise the
maximum relative error |p(f) / 2^f - 1| on [-1/2, 1/2].

Method: Lawson's algorithm (iteratively reweighted least squares converging
to the minimax solution; C. L. Lawson, "Contributions to the theory of linear
least maximum approximation", 1961) on a dense grid, in float64.  Then the
coefficients are rounded to float32, and the error of the float32 Horner
evaluation (one rounding per fused multiply-add) is measured on a dense grid.

    python fit_exp2_poly.py [DEG]      # prints coefficients and errors
"""
from __future__ import annotations

import sys

import numpy as np


def lawson_fit(deg: int, n: int = 20001, iters: int = 400) -> np.ndarray:
    f = np.cos(np.linspace(0.0, np.pi, n)) * 0.5          # Chebyshev-clustered grid on [-1/2, 1/2]
    target = np.exp2(f)
    A = np.vander(f, deg + 1, increasing=True) / target[:, None]   # relative-error design
    b = np.ones_like(f)
    w = np.full(n, 1.0 / n)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    return c


def horner_f32(c32: np.ndarray, f: np.ndarray) -> np.ndarray:
    """p(f) in float32 with one rounding per fma (emulated exactly in float64)."""
    f = f.astype(np.float32)
    acc = np.full_like(f, c32[-1])
    for ck in c32[-2::-1]:
        acc = (acc.astype(np.float64) * f.astype(np.float64) + np.float64(ck)).astype(np.float32)
    return acc


def report(deg: int):
    c = lawson_fit(deg)
    c32 = c.astype(np.float32)
    f = np.linspace(-0.5, 0.5, 2_000_001)
    rel64 = np.abs(np.polyval(c[::-1], f) / np.exp2(f) - 1).max()
    rel32 = np.abs(horner_f32(c32, f).astype(np.float64) / np.exp2(f.astype(np.float32).astype(np.float64)) - 1).max()
    return c32, rel64, rel32


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 5
    c32, rel64, rel32 = report(deg)
    print("degree %d: max rel err %.3g (exact coeffs), %.3g (float32 Horner)" % (deg, rel64, rel32))
    for k, ck in enumerate(c32):
        print("  c%d = %s  (%s)" % (k, np.format_float_scientific(ck, unique=True), float(ck).hex()))
