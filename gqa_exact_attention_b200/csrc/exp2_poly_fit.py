"""Fit of the exp2 polynomial in exp2_poly.cuh.

Finds c1, c2, c3 minimising max |(1 + c1 f + c2 f^2 + c3 f^3) / 2^f - 1| over f in
[-1/2, 1/2] (the constant term held at 1), as a linear program over a dense grid, and
prints the coefficients rounded to float32 with the float32-evaluated error.
"""
import numpy as np


def fit(n_grid: int = 4001):
    from scipy.optimize import linprog
    f = np.linspace(-0.5, 0.5, n_grid)
    y = 2.0 ** f
    A = np.stack([f, f ** 2, f ** 3], 1)
    # |1 + A c - y| <= e y  <=>  A c - e y <= y - 1  and  -A c - e y <= 1 - y
    a_ub = np.vstack([np.hstack([A, -y[:, None]]), np.hstack([-A, -y[:, None]])])
    b_ub = np.concatenate([y - 1.0, 1.0 - y])
    r = linprog([0, 0, 0, 1], A_ub=a_ub, b_ub=b_ub, bounds=[(None, None)] * 4, method="highs")
    assert r.success, r.message
    return np.float32(r.x[:3]), float(r.x[3])


if __name__ == "__main__":
    c, err = fit()
    print("c1, c2, c3 =", [float(x) for x in c], "minimax relative error", err)
