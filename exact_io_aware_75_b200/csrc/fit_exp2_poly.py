"""Fit the cubic used by the prefill kernel's software exponential.

2^x is split as 2^floor(x) * 2^f with f in [0, 1); 2^floor(x) is placed by an
integer add into the float's exponent bits, and 2^f is this cubic
p(f) = c0 + c1 f + c2 f^2 + c3 f^3, chosen to minimise the maximum relative
error max |p(f) / 2^f - 1| over [0, 1] (a linear program on a dense grid),
with p(0) = 1 exactly so that a score equal to the row max maps to 1.

    python exact_io_aware_75_b200/csrc/fit_exp2_poly.py

prints the coefficients (as fp32 hex) and the error of the fp32 evaluation.
"""
import numpy as np
from scipy.optimize import linprog


def fit(degree=3, n=4001):
    f = np.linspace(0.0, 1.0, n)
    t = np.exp2(f)
    # unknowns: c1..c_deg, e   (c0 fixed to 1)
    A, b = [], []
    for fi, ti in zip(f, t):
        row = [fi ** k / ti for k in range(1, degree + 1)]
        # (1 + sum c_k f^k)/t - 1 <= e   and   -(...) + 1 <= e
        A.append(row + [-1.0]); b.append(1.0 - 1.0 / ti)
        A.append([-r for r in row] + [-1.0]); b.append(-(1.0 - 1.0 / ti))
    c = np.zeros(degree + 1); c[-1] = 1.0
    res = linprog(c, A_ub=np.array(A), b_ub=np.array(b), bounds=[(None, None)] * (degree + 1))
    assert res.success
    return np.concatenate([[1.0], res.x[:degree]]), res.x[degree]


def eval_fp32(coef, x):
    """The kernel's evaluation, in fp32 (numpy float32 arithmetic)."""
    x = np.maximum(x.astype(np.float32), np.float32(-127.0))
    j = np.floor(x).astype(np.float32)
    f = (x - j).astype(np.float32)
    c = coef.astype(np.float32)
    p = np.float32(c[3])
    p = (p * f + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    bits = p.view(np.uint32).astype(np.int64) + (j.astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    coef, err = fit()
    c32 = coef.astype(np.float32)
    print("minimax relative error (real arithmetic): %.3e" % err)
    for k, v in enumerate(c32):
        print("c%d = %.9e  (0x%08x)" % (k, v, np.float32(v).view(np.uint32)))
    x = np.linspace(-126.0, 8.0, 2_000_001)
    rel = np.abs(eval_fp32(coef, x).astype(np.float64) / np.exp2(x) - 1.0)
    print("fp32 evaluation, x in [-126, 8]: max relative error %.3e" % rel.max())
