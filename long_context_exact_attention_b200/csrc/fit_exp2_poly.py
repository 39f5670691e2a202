"""Fits the polynomial the forward kernel uses to evaluate part of its
exponentials on the FMA pipe instead of the MUFU unit.

Method (Cody-Waite style range reduction, minimax fit by Lawson's
iteratively reweighted least squares):
    2^x = 2^floor(x) * 2^f,  f = x - floor(x) in [0, 1)
    2^f ~= c0 + c1 f + c2 f^2 + c3 f^3   (minimax in RELATIVE error on [0,1))
The integer part is added to the float's exponent field.  The constraint
c0 = 1 keeps 2^n exact at integers.  Run from the repository root:
    python long_context_exact_attention_b200/csrc/fit_exp2_poly.py
It prints the coefficients (float32) and the relative error bound; the
numbers in exp2_poly.cuh come from this script.
"""

import numpy as np


def fit(degree=3, iters=200, n=20001):
    f = np.linspace(0.0, 1.0, n)
    target = np.exp2(f)
    # basis without the constant term (c0 fixed to 1): relative residual
    A = np.stack([f ** k for k in range(1, degree + 1)], axis=1) / target[:, None]
    b = (target - 1.0) / target
    w = np.ones(n)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        r = np.abs(A @ c - b)
        w = w * (r + 1e-30)
        w /= w.sum()
    coef = np.concatenate([[1.0], c]).astype(np.float32)
    return coef


def rel_error(coef, n=200001):
    f = np.linspace(0.0, 1.0, n, dtype=np.float64)
    p = np.polyval(coef[::-1].astype(np.float64), f)
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit()
    print("coefficients (c0..c3):", [float(x) for x in c])
    print("float32 hex:", [hex(np.float32(x).view(np.uint32)) for x in c])
    print("max relative error on [0,1):", rel_error(c))
