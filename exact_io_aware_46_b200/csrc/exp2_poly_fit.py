"""Fits the coefficients of the software 2^f used by the forward softmax.

Method: Cody-Waite style range reduction x = n + f with n = round(x) and
f in [-1/2, 1/2], then 2^x = 2^n * q(f) where q is the degree-DEG polynomial
minimising the maximum *relative* error max |q(f) / 2^f - 1| over f in
[-1/2, 1/2] (a minimax fit, solved here as a linear programme on a dense
grid rather than by Remez exchange).  The constant term is pinned to 1 so that
2^0 = 1 exactly.  Run: python exp2_poly_fit.py [degree]
"""

import sys

import numpy as np
from scipy.optimize import linprog


def fit(deg: int, n: int = 4001):
    f = np.linspace(-0.5, 0.5, n)
    t = np.exp2(f)
    # unknowns: c1..c_deg, e ; minimise e s.t. |1 + sum c_k f^k - t| <= e t
    A = np.stack([f ** k for k in range(1, deg + 1)], axis=1)
    rhs = t - 1.0
    ones = t[:, None]
    A_ub = np.block([[A, -ones], [-A, -ones]])
    b_ub = np.concatenate([rhs, -rhs])
    c = np.zeros(deg + 1)
    c[-1] = 1.0
    res = linprog(c, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * (deg + 1), method="highs")
    coef = np.concatenate([[1.0], res.x[:deg]])
    return coef, res.x[deg]


def eval_f32(coef, x):
    """The kernel's steps in fp32: round-to-nearest reduction by the 1.5*2^23
    trick, Horner in fp32 (FMA), exponent insertion by integer add."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-127.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = t.view(np.int32) - np.int32(0x4B400000)
    f = (x - (t - magic)).astype(np.float32)
    c = [np.float32(v) for v in coef]
    p = np.float32(c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (np.float64(p) * f + c[k]).astype(np.float32)  # fma: one rounding
    return (p.view(np.int32) + (n << 23)).view(np.float32)


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    coef, err = fit(deg)
    print(f"degree {deg}: max relative error {err:.3e}")
    for k, v in enumerate(coef):
        print(f"  c{k} = {np.float32(v)!r}  ({v:.10e})")
    x = np.linspace(-126, 0, 2000001, dtype=np.float32)
    y = eval_f32(coef, x)
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)
    print(f"  fp32 evaluation on [-126, 0]: max rel error {rel.max():.3e}")
