"""Derives the coefficients of the degree-4 polynomial p(f) ~ 2^f, f in [-1/2, 1/2],
that the attention kernel uses for part of its exponentials (exp2_poly in
ptx.cuh).  Method: least squares on a dense grid, re-weighted repeatedly
toward the points of largest relative error (an iterative approach to the
minimax polynomial); then the fp32 Horner evaluation is checked.

    python fit_exp2_poly.py   ->  max relative error 2.68e-06 and the coefficients
"""
import numpy as np


def fit(deg=4, iters=60):
    f = np.linspace(-0.5, 0.5, 20001)
    y = 2.0 ** f
    w = 1 / y
    V = np.vander(f, deg + 1, increasing=True)
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(V * w[:, None], y * w, rcond=None)
        err = (V @ c - y) / y
        w = w * (1 + 50 * np.abs(err) / np.abs(err).max())
    c32 = c.astype(np.float32)
    ff = f.astype(np.float32)
    p = np.float32(c32[-1])
    for k in range(deg - 1, -1, -1):
        p = (p * ff + c32[k]).astype(np.float32)
    return c32, float((np.abs(p.astype(np.float64) - y) / y).max())


if __name__ == "__main__":
    c, e = fit()
    print(f"max relative error {e:.3e}")
    for k, v in enumerate(c):
        print(f"c{k} = {float(v)!r}")
