"""Coefficients of the FMA-pipe exp2 used by the attention kernel's softmax.

The kernel evaluates part of its 2^x terms without the special-function unit, by Cody-Waite
range reduction (W. J. Cody and W. Waite, "Software Manual for the Elementary Functions", 1980):
x = n + f with n = round(x) and f in [-1/2, 1/2], 2^x = 2^n * 2^f, where 2^n goes straight into
the exponent field and 2^f comes from a polynomial

    p(f) = 1 + c1 f + c2 f^2 + c3 f^3,

whose constant term is pinned to exactly 1 (so that a clamped argument of -127 yields +0.0).
c1..c3 minimise the maximum relative error max |p(f) / 2^f - 1| over [-1/2, 1/2] (a discrete
minimax fit, solved as a linear programme on a dense grid), then are rounded to fp32.

Run as a script to print the fit; `tests/test_exp2_poly.py` checks that the constants in the CUDA
source stay within the error bound this fit achieves.
"""

from __future__ import annotations

import numpy as np


def fit(degree: int = 3, grid: int = 4001) -> tuple[np.ndarray, float]:
    """Minimax relative-error fit of 2^f on [-1/2, 1/2] with p(0) = 1; returns (c1..c_deg, err)."""
    from scipy.optimize import linprog

    f = np.linspace(-0.5, 0.5, grid)
    y = np.exp2(f)
    # relative error of p at f:  (1 + sum_k c_k f^k) / y - 1  =  A c - b
    A = np.stack([f ** k / y for k in range(1, degree + 1)], axis=1)
    b = (y - 1.0) / y
    ones = np.ones((grid, 1))
    a_ub = np.vstack([np.hstack([A, -ones]), np.hstack([-A, -ones])])
    b_ub = np.concatenate([b, -b])
    cost = np.r_[np.zeros(degree), 1.0]
    res = linprog(cost, A_ub=a_ub, b_ub=b_ub,
                  bounds=[(None, None)] * degree + [(0.0, None)], method="highs")
    if not res.success:
        raise RuntimeError(res.message)
    return res.x[:degree], float(res.x[degree])


if __name__ == "__main__":
    c, err = fit()
    c32 = c.astype(np.float32)
    print(f"max relative error of the real-coefficient fit: {err:.3e}")
    for k, v in enumerate(c32, start=1):
        print(f"c{k} = {float(v).hex()}f  // {float(v):.9g}")
