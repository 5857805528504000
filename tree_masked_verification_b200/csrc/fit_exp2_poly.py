"""Fit of the cubic used for part of the exp2 evaluations in prefix_tc.cu.

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]; 2^f is
approximated by c0 + c1 f + c2 f^2 + c3 f^3.  The coefficients minimise the
largest relative error over [-1/2, 1/2] (Lawson's iteratively reweighted
least squares on a dense grid), then are rounded to fp32; the printed error
is that of the fp32 coefficients.  A relative error of 7.5e-5 is far below
half an ulp of bf16 (2^-9), the precision P is stored in.

    python fit_exp2_poly.py
"""
import numpy as np


def fit(degree=3, points=20001, iters=200):
    f = np.linspace(-0.5, 0.5, points)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)
    w = np.ones_like(f)
    for _ in range(iters):
        sw = np.sqrt(w) / y
        c, *_ = np.linalg.lstsq(V * sw[:, None], y * sw, rcond=None)
        err = np.abs(V @ c - y) / y
        w = w * err
        w /= w.sum()
    c32 = c.astype(np.float32)
    err32 = np.max(np.abs(V @ c32.astype(np.float64) - y) / y)
    return c32, err32


if __name__ == "__main__":
    c, e = fit()
    for i, v in enumerate(c):
        print(f"c{i} = {float(v)!r}")
    print(f"max relative error {e:.3g}")
