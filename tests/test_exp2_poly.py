"""The forward's software 2^x (FMA pipe) against the exact exponential.

The constants are read from the CUDA source, so this pins what the kernel
uses: Cody-Waite reduction with round-to-nearest, degree-3 minimax
polynomial, exponent insertion.  The bound (1.02e-4 relative) is far below the
bf16 rounding of P (2^-9 = 1.95e-3 relative)."""

import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_io_aware_46_b200", "csrc")


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "sm100.cuh")).read()
    body = src[src.index("ex2_poly2(float2 x_in)"):]
    body = body[:body.index("\n}\n")]
    c3, c2 = re.search(r"__ffma2_rn\(make_float2\(([0-9.e-]+)f, \1f\), f,\s*make_float2\(([0-9.e-]+)f",
                       body).groups()
    c1 = re.search(r"q = __ffma2_rn\(q, f, make_float2\(([0-9.e-]+)f", body).group(1)
    return [1.0, float(c1), float(c2), float(c3)]


def test_polynomial_error_bound():
    sys.path.insert(0, CSRC)
    from exp2_poly_fit import eval_f32

    coef = _kernel_coefficients()
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32)
    y = eval_f32(coef, x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 1.02e-4
    # integers are exact up to the polynomial's value at f = 0 (c0 = 1)
    xi = np.arange(-125, 9, dtype=np.float32)
    assert np.array_equal(eval_f32(coef, xi), np.exp2(xi))


def test_refit_reproduces_kernel_constants():
    sys.path.insert(0, CSRC)
    from exp2_poly_fit import fit

    coef, err = fit(3)
    assert err <= 1.02e-4
    assert np.allclose(np.float32(coef), np.float32(_kernel_coefficients()), rtol=1e-6)
