"""Fits the polynomial used by exp2_poly_x2 (common.cuh): 2^f on [-0.5, 0.5],
degree 4, minimising the maximum relative error by Lawson's iteratively
reweighted least squares.  Prints the coefficients (c0..c4) and the max
relative error of the fp32 Horner evaluation.

    python blockwise_exact_attention_block_b200/csrc/fit_exp2_poly.py
"""
import numpy as np


def fit(deg=4, iters=200):
    f = np.linspace(-0.5, 0.5, 20001)
    y = np.exp2(f)
    V = np.vander(f, deg + 1, increasing=True)
    w = np.ones_like(f)
    for _ in range(iters):
        W = w / y
        c, *_ = np.linalg.lstsq(V * W[:, None], y * W, rcond=None)
        err = (V @ c - y) / y
        w = w * np.abs(err) ** 0.5 + 1e-30
        w /= w.sum()
    cf = c.astype(np.float32)
    ff = f.astype(np.float32)
    p = np.full_like(ff, cf[-1])
    for k in range(deg - 1, -1, -1):
        p = p * ff + cf[k]
    return cf, float(np.max(np.abs(p.astype(np.float64) - y) / y))


if __name__ == "__main__":
    cf, e = fit()
    print("coefficients:", [f"{float(x):.9e}" for x in cf])
    print("max relative error (fp32 Horner):", e)
