"""Fit of the degree-3 polynomial for 2^f, f in [-1/2, 1/2], used by exp2_poly2 in sm100.cuh.

The attention kernels evaluate part of the softmax's exponentials on the FMA
pipe: x = n + f with n = round(x), 2^x = 2^n * p(f). This script finds the p
of degree 3 whose largest RELATIVE error |p(f)/2^f - 1| on [-1/2, 1/2] is as
small as it can be, by Lawson's iteratively reweighted least squares:
solve a weighted least-squares fit of p(f)/2^f to 1 on a dense grid, multiply
each point's weight by its current error, renormalise, repeat. The weights
concentrate on the points of largest error and the fit converges to the
minimax polynomial, whose error equioscillates at degree + 2 = 5 points
(Chebyshev's alternation theorem).

    python reduced_query_head_b200/csrc/fit_exp2_poly.py

prints the four coefficients (constant term first) and the maximum relative
error; sm100.cuh holds them as float literals.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3


def fit(grid_points: int = 4001, iterations: int = 2000):
    """Coefficients c[0..3] (p(f) = c0 + c1 f + c2 f^2 + c3 f^3) and their max relative error."""
    f = np.linspace(-0.5, 0.5, grid_points)
    y = np.exp2(f)
    a = np.vander(f, DEGREE + 1, increasing=True)
    w = np.full(f.shape, 1.0 / f.size)
    c = None
    for _ in range(iterations):
        sw = np.sqrt(w)
        # minimise sum_k w_k (p(f_k) / y_k - 1)^2
        c, *_ = np.linalg.lstsq(a * (sw / y)[:, None], sw, rcond=None)
        err = np.abs(a @ c / y - 1.0)
        w = w * err
        w /= w.sum()
    err = float(np.max(np.abs(a @ c / y - 1.0)))
    return c, err


if __name__ == "__main__":
    coef, max_rel = fit()
    print("c0..c3 =", ", ".join(repr(float(x)) for x in coef))
    print("max relative error on [-1/2, 1/2] = %.4e" % max_rel)
