"""Derives the cubic used by the prefill kernel for 2^x on the FMA pipe.

The kernel splits x = j + f with j = round(x) and f in [-1/2, 1/2], evaluates
2^f by a cubic c0 + c1 f + c2 f^2 + c3 f^3 and adds j to the exponent field.
The coefficients minimise the maximum relative error of the cubic on
[-1/2, 1/2]; they are found here by Lawson's algorithm (iteratively reweighted
least squares) in float64 and then rounded to float32.

    python -m rope_frequency_sparse_b200.exp2_poly_fit

prints the four coefficients and the error of the float32 evaluation that the
kernel performs (range reduction by the 1.5 * 2^23 rounding constant, Horner in
fp32, integer add of j << 23), over x in [-125, 9] (every result a normal
float; at the clamp x = -126 itself the result is subnormal and ~1e-38).
"""
from __future__ import annotations

import numpy as np

ROUND_MAGIC = np.float32(12582912.0)  # 1.5 * 2^23


def fit_coefficients(degree: int = 3, iterations: int = 400, points: int = 20001) -> np.ndarray:
    """Minimax-relative-error polynomial for 2^f on [-1/2, 1/2] (Lawson), as float32."""
    f = np.linspace(-0.5, 0.5, points)
    y = np.exp2(f)
    a = np.vander(f, degree + 1, increasing=True) / y[:, None]
    b = np.ones_like(f)
    w = np.full(points, 1.0 / points)
    c = None
    for _ in range(iterations):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(a * sw[:, None], b * sw, rcond=None)
        e = np.abs(a @ c - b)
        w = w * e
        w /= w.sum()
    return c.astype(np.float32)


def exp2_fp32(x: np.ndarray, coeffs: np.ndarray) -> np.ndarray:
    """The kernel's evaluation of 2^x, step for step in float32 (x clamped at -126)."""
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    t = (x + ROUND_MAGIC).astype(np.float32)
    f = (x - (t - ROUND_MAGIC).astype(np.float32)).astype(np.float32)
    c0, c1, c2, c3 = (np.float32(v) for v in coeffs)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + c0).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + ((t.view(np.uint32).astype(np.uint64) << 23) & 0xFFFFFFFF))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def max_relative_error(coeffs: np.ndarray, lo: float = -126.0, hi: float = 9.0, n: int = 2000001) -> float:
    x = np.linspace(lo, hi, n).astype(np.float32)
    got = exp2_fp32(x, coeffs).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(got / ref - 1.0)))


if __name__ == "__main__":
    c = fit_coefficients()
    print("c0..c3 =", ", ".join(repr(float(v)) for v in c))
    print("max relative error over x in [-125, 9]: %.3e" % max_relative_error(c, -125.0, 9.0))
