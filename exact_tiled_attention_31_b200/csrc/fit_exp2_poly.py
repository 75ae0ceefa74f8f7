"""Fit the polynomial used for 2^f, f in [-1/2, 1/2], by the forward kernel.

Method (Cody & Waite style range reduction): 2^x = 2^j * 2^f with j the
nearest integer to x and f = x - j in [-1/2, 1/2].  2^f is approximated by
p(f) = 1 + c1 f + c2 f^2 + c3 f^3 (the constant term is pinned to 1 so that
p(0) = 1 exactly: a row's largest probability, 2^0, stays exactly 1).  The
coefficients minimise the maximum relative error: a weighted least-squares fit
on Chebyshev nodes, re-weighted (Lawson's iteration) towards the minimax
solution.  Run this file to regenerate the constants and their error bound.
"""
import numpy as np


def fit(deg: int = 3, iters: int = 200):
    n = 2001
    f = 0.5 * np.cos(np.pi * (np.arange(n) + 0.5) / n)  # Chebyshev nodes on [-1/2, 1/2]
    target = np.exp2(f)
    A = np.stack([f ** k for k in range(1, deg + 1)], axis=1) / target[:, None]
    b = (target - 1.0) / target
    w = np.ones(n) / n
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    return c


def max_rel_err(c):
    f = np.linspace(-0.5, 0.5, 200001)
    p = 1.0 + sum(ck * f ** (k + 1) for k, ck in enumerate(c))
    return np.abs(p / np.exp2(f) - 1.0).max()


if __name__ == "__main__":
    c = fit()
    c32 = np.float32(c)
    print("coefficients (fp32):", [float(x) for x in c32])
    print("max relative error on [-1/2, 1/2]: %.3e" % max_rel_err(c32.astype(np.float64)))
