"""Derives the coefficients of the polynomial exp2 used by the reduced-attention
softmax kernel (``exp2_poly2`` in csrc/sm100.cuh).

Method: range reduction to 2^x = 2^j * 2^f with j = round(x) and
f = x - j in [-1/2, 1/2], then 2^f by the degree-3 polynomial with p(0) = 1
whose maximum relative error over [-1/2, 1/2] is smallest (a minimax /
Chebyshev fit, solved here as a linear program over a dense grid of f:
minimise t subject to |p(f_i) 2^-f_i - 1| <= t).  The coefficients are
rounded to fp32 and the error of the rounded polynomial, evaluated in fp32 with fused multiply-adds
in Horner order as the kernel does, is reported.

Run:  python token_skipping_sparse_b200/exp2_poly_fit.py
"""

from __future__ import annotations

import numpy as np
from scipy.optimize import linprog

DEGREE = 3


def fit(degree=DEGREE, n=4001):
    """Minimax relative-error fit with p(0) = 1 exactly: then an input
    clamped at -127 (j = -127, f = 0) gives the bits of 1.0 plus -127 in the
    exponent field, i.e. exactly +0, so masked scores (-inf) vanish."""
    f = np.linspace(-0.5, 0.5, n)
    w = 2.0 ** -f                                   # relative error: p(f) / 2^f - 1
    V = np.vander(f, degree + 1, increasing=True)[:, 1:]   # columns f^1 .. f^degree (c_0 = 1)
    # variables: c_1..c_degree, t ; minimise t subject to |(1 + V c) w - 1| <= t
    c_obj = np.zeros(degree + 1)
    c_obj[-1] = 1.0
    A = np.vstack([np.hstack([V * w[:, None], -np.ones((n, 1))]),
                   np.hstack([-V * w[:, None], -np.ones((n, 1))])])
    b = np.concatenate([1.0 - w, w - 1.0])
    res = linprog(c_obj, A_ub=A, b_ub=b, bounds=[(None, None)] * degree + [(0, None)], method="highs")
    assert res.success, res.message
    return np.concatenate([[1.0], res.x[:-1]]), res.x[-1]


def horner_fp32(c, f):
    c = np.asarray(c, dtype=np.float32)
    f = np.asarray(f, dtype=np.float32)
    p = np.full_like(f, c[-1])
    for a in c[-2::-1]:
        p = (p.astype(np.float64) * f + a).astype(np.float32)    # one rounding per step, as an FMA
    return p


if __name__ == "__main__":
    c, t = fit()
    c32 = c.astype(np.float32)
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float32)
    err = np.abs(horner_fp32(c32, f).astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0).max()
    print(f"degree {DEGREE}: minimax relative error {t:.3e}; fp32 Horner {err:.3e}")
    for i, a in enumerate(c32):
        print(f"  c{i} = {float(a)!r}f  ({float(a).hex()})")
