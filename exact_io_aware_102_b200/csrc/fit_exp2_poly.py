"""Fit the degree-3 polynomial for 2^f on [-1/2, 1/2] used by the FMA-pipe
exponential in attn_fwd.cu (ex2_poly2).

Iteratively reweighted least squares on Chebyshev nodes, minimising the
relative error; prints the float32 coefficients c0..c3 and the max relative
error of the rounded coefficients (7.5e-5).
"""
import numpy as np


def fit(degree=3, nodes=4001, rounds=30):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)
    y = 2.0 ** f
    V = np.vander(f, degree + 1, increasing=True)
    w = 1.0 / y
    c = np.linalg.lstsq(V * w[:, None], y * w, rcond=None)[0]
    for _ in range(rounds):
        r = (V @ c - y) / y
        w = w * (1 + 50 * np.abs(r) / np.abs(r).max())
        c = np.linalg.lstsq(V * w[:, None], y * w, rcond=None)[0]
    return c.astype(np.float32)


if __name__ == "__main__":
    c = fit()
    x = np.linspace(-0.5, 0.5, 200001)
    rel = np.abs(np.polyval(c.astype(np.float64)[::-1], x) / 2.0 ** x - 1).max()
    print("c0..c3 =", ", ".join("%.8gf" % v for v in c), " max rel err = %.3g" % rel)
