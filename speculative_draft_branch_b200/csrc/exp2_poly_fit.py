"""Provenance of the exp2 polynomial coefficients in sm100.cuh (not run at
build time).

2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (range
reduction in the style of Cody and Waite).  2^f is approximated by a cubic
fitted here by Lawson's iteratively reweighted least squares, which converges
to the minimax (equal-ripple) polynomial for the relative error.  Printed:
coefficients c0..c3 rounded to fp32 and the max relative error of the fp32
Horner evaluation on a dense grid (about 7.5e-5).
"""
import numpy as np


def fit(deg=3, iters=60):
    f = np.cos(np.linspace(0, np.pi, 20001)) * 0.5
    y = 2.0 ** f
    w = 1.0 / y
    for _ in range(iters):
        A = np.vander(f, deg + 1, increasing=True) * w[:, None]
        c, *_ = np.linalg.lstsq(A, y * w, rcond=None)
        err = (np.polyval(c[::-1], f) - y) / y
        w = w * (np.abs(err) / np.abs(err).max() + 1e-3) ** 0.5
        w /= w.max()
    c32 = c.astype(np.float32)
    ff = np.linspace(-0.5, 0.5, 2000001).astype(np.float32)
    p = np.float32(c32[deg])
    for k in range(deg - 1, -1, -1):
        p = (p * ff + c32[k]).astype(np.float32)
    rel = np.abs(p.astype(np.float64) / 2.0 ** ff.astype(np.float64) - 1).max()
    return c32, rel


if __name__ == "__main__":
    c, rel = fit()
    print("coefficients:", [float(x) for x in c], "max relative error:", rel)
