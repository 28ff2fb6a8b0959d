"""Fits the cubic that ex2_poly2 (common.cuh) uses for 2^f on [-1/2, 1/2].

p(f) = 1 + c1 f + c2 f^2 + c3 f^3 with the constant term fixed at 1 (so that
2^0 is exactly 1, and the clamped argument -127 maps to the bit pattern of 0),
chosen to minimise the largest relative
error |p(f) / 2^f - 1| over a dense grid: a small linear programme in
(c1, c2, c3, e). Prints the coefficients rounded to fp32 and the largest
relative error of fp32 Horner evaluation with them.

    python block_sparse_long_04_b200/csrc/fit_exp2_poly.py
"""
import numpy as np
from scipy.optimize import linprog


def fit(deg: int = 3, n_grid: int = 4001):
    f = np.linspace(-0.5, 0.5, n_grid)
    t = np.exp2(f)
    A = np.stack([f ** k / t for k in range(1, deg + 1)], 1)   # (p - 1) / 2^f, per coefficient
    b0 = 1.0 / t - 1.0
    ones = np.ones((n_grid, 1))
    A_ub = np.vstack([np.hstack([A, -ones]), np.hstack([-A, -ones])])
    b_ub = np.concatenate([-b0, b0])
    res = linprog(np.r_[np.zeros(deg), 1.0], A_ub=A_ub, b_ub=b_ub,
                  bounds=[(None, None)] * (deg + 1))
    c = res.x[:deg].astype(np.float32)
    ff = f.astype(np.float32)
    p = np.float32(c[-1])
    for k in range(deg - 2, -1, -1):
        p = p * ff + c[k]
    p = p * ff + np.float32(1.0)
    return c, float(np.max(np.abs(p.astype(np.float64) / t - 1.0)))


if __name__ == "__main__":
    c, err = fit()
    for k, v in enumerate(c, 1):
        print(f"c{k} = {float(v)!r}f  // {float(v).hex()}")
    print(f"max relative error (fp32 Horner) = {err:.3e}")
