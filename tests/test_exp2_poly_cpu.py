"""The prefill kernel evaluates part of its softmax exponentials on the FMA pipe
(round-to-nearest split, cubic for 2^f, exponent-field add).  These CPU checks pin
the constants compiled into the kernel: they are re-read from the CUDA source,
re-derived by the fitting script, and the kernel's float32 evaluation is held to
its error bound against the exact 2^x over the whole input range it sees."""
import os
import re

import numpy as np
import pytest

from rope_frequency_sparse_b200 import exp2_poly_fit

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "rope_frequency_sparse_b200", "csrc", "prefill_tc.cu")


def kernel_coefficients():
    text = open(SRC).read()
    vals = []
    for k in range(4):
        m = re.search(rf"constexpr float kExpC{k} = ([0-9.eE+-]+)f;", text)
        assert m, f"kExpC{k} not found"
        vals.append(np.float32(float(m.group(1))))
    return np.array(vals, dtype=np.float32)


def test_coefficients_are_the_fit():
    # the fit is deterministic; the kernel must carry its float32 rounding
    assert np.array_equal(kernel_coefficients(), exp2_poly_fit.fit_coefficients())


def test_relative_error_bound_over_kernel_range():
    # x = s * scale - m_ref lies in [-inf, 8 + rounding]; the kernel clamps at -126.
    # Down to -125 every result is a normal float; at the clamp itself (2^-126, the
    # smallest normal) a cubic value below 1 lands on a subnormal and loses ~1e-4
    # relative, which is harmless at 1e-38 (see test_clamp_underflows_to_tiny).
    err = exp2_poly_fit.max_relative_error(kernel_coefficients(), -125.0, 9.0)
    assert err < 1e-4          # far below bf16 rounding of P (2^-9 ~ 2e-3)


@pytest.mark.parametrize("x", [0.0, 1.0, -1.0, 0.5, -0.5, 8.0, -20.25, -125.5])
def test_exact_points(x):
    got = float(exp2_poly_fit.exp2_fp32(np.array([x], dtype=np.float32), kernel_coefficients())[0])
    assert abs(got / 2.0 ** x - 1.0) < 1e-4


def test_integer_part_enters_the_exponent():
    # for x = j + f the result must scale by exactly 2^j: a dropped or mis-shifted
    # exponent add shows up as a factor of 2^k
    c = kernel_coefficients()
    f = np.linspace(-0.49, 0.49, 99, dtype=np.float32)
    base = exp2_poly_fit.exp2_fp32(f, c).astype(np.float64)
    for j in (-100, -7, -1, 1, 5, 8):
        got = exp2_poly_fit.exp2_fp32(f + np.float32(j), c).astype(np.float64)
        assert np.allclose(got, base * 2.0 ** j, rtol=1e-6)


def test_clamp_underflows_to_tiny():
    # masked logits reach the exponential as -inf: the clamp keeps a valid tiny value
    got = exp2_poly_fit.exp2_fp32(np.array([-np.inf, -1e30, -200.0], dtype=np.float32), kernel_coefficients())
    assert np.all(np.isfinite(got)) and np.all(got >= 0) and np.all(got < 1.2e-38)
