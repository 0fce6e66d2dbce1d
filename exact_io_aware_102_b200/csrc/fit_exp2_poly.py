"""Fit the degree-3 polynomial for 2^f on [-1/2, 1/2] used by the FMA-pipe
exponential in attn_fwd.cu (ex2_poly2 in sm100_ptx.cuh).

The constant term is fixed at exactly 1, so that 2^f is exact at f = 0: the
kernel clamps its argument at -127, where the polynomial must give exactly 1
for the result's exponent field to come out as exactly 0 (a masked score then
yields +0).  The other three coefficients minimise the maximum relative error
on a dense grid (a linear program, minimax), then are rounded to float32.
Run as a script it prints c1..c3 and the max relative error of the rounded
coefficients (1.013e-4).
"""
import numpy as np

GRID = 20001


def fit(grid=GRID):
    """float32 [c0 = 1, c1, c2, c3] minimising max |q(f) / 2^f - 1| over f in [-1/2, 1/2]."""
    from scipy.optimize import linprog
    f = np.linspace(-0.5, 0.5, grid)
    y = 2.0 ** f
    # unknowns c1, c2, c3, t; minimise t subject to |(1 + c1 f + c2 f^2 + c3 f^3) / y - 1| <= t
    a = np.stack([f / y, f ** 2 / y, f ** 3 / y], 1)
    b = 1.0 / y - 1.0
    ones = np.ones((grid, 1))
    a_ub = np.vstack([np.hstack([a, -ones]), np.hstack([-a, -ones])])
    b_ub = np.concatenate([-b, b])
    res = linprog([0.0, 0.0, 0.0, 1.0], A_ub=a_ub, b_ub=b_ub, bounds=[(None, None)] * 3 + [(0, None)],
                  method="highs")
    if not res.success:
        raise RuntimeError(res.message)
    return np.concatenate([[1.0], res.x[:3]]).astype(np.float32)


def max_rel_error(c, points=400001):
    """Max relative error of the polynomial with coefficients c (evaluated in fp64) on [-1/2, 1/2]."""
    x = np.linspace(-0.5, 0.5, points)
    return float(np.abs(np.polyval(np.asarray(c, np.float64)[::-1], x) / 2.0 ** x - 1).max())


if __name__ == "__main__":
    c = fit()
    print("c0..c3 =", ", ".join("%.8gf" % v for v in c), " max rel err = %.4g" % max_rel_error(c))
