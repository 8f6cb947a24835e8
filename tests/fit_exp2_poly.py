"""Fits the cubic that the forward kernel uses to evaluate part of its exp2 calls on the FMA
pipe instead of the special-function unit.

Method: range reduction x = j + f with j = round(x) (so f in [-1/2, 1/2]) and 2^x = 2^j * 2^f;
2^j is applied by adding j to the exponent field.  2^f is approximated by
p(f) = 1 + c1 f + c2 f^2 + c3 f^3 (constant term fixed at 1, so 2^0 is exact and the row
maximum keeps probability exactly 1).  c1..c3 minimise the maximum relative error on
[-1/2, 1/2]: a least-squares start on Chebyshev nodes, then Lawson's iteratively re-weighted
least squares toward the minimax solution.  Run this module to print the coefficients, their
float32 values and the achieved error.
"""

from __future__ import annotations

import numpy as np


def fit(degree: int = 3, iters: int = 200):
    n = 4000
    f = 0.5 * np.cos(np.pi * (np.arange(n) + 0.5) / n)          # Chebyshev nodes on [-1/2, 1/2]
    target = np.exp2(f)
    A = np.stack([f ** k for k in range(1, degree + 1)], axis=1) / target[:, None]
    b = (target - 1.0) / target                                  # relative residual, c0 = 1
    w = np.ones(n) / n
    c = None
    for _ in range(iters):                                       # Lawson: reweight by |error|
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        e = np.abs(A @ c - b)
        w = w * e
        w /= w.sum()
    return c


def max_rel_error(c, fp32: bool = True):
    f = np.linspace(-0.5, 0.5, 200001)
    if fp32:
        f = f.astype(np.float32)
        cc = [np.float32(x) for x in c]
        p = np.float32(1.0)
        acc = cc[-1]
        for k in range(len(cc) - 2, -1, -1):
            acc = acc * f + cc[k]
        p = acc * f + np.float32(1.0)
        return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))
    p = 1.0 + sum(ci * f ** (k + 1) for k, ci in enumerate(c))
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit()
    print("coefficients c1..c3:", ", ".join(f"{x:.9e}" for x in c))
    print("as float32:         ", ", ".join(f"{np.float32(x).item():.9e}f" for x in c))
    print(f"max relative error (exact arithmetic): {max_rel_error(c, fp32=False):.3e}")
    print(f"max relative error (fp32 Horner):      {max_rel_error(c, fp32=True):.3e}")
