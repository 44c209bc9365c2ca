"""Derive the cubic used for 2^f, f in [-0.5, 0.5], by the prefill kernel's
FMA-pipe exponential (csrc/sm100_ptx.cuh, exp2_poly_f2).

Minimax fit of the relative error, solved as a linear program on a dense grid:
minimise e subject to |p(f_i) - 2^f_i| <= e * 2^f_i. Prints the coefficients
(as float32 hex literals, the form used in the kernel) and the error bound.
Run: python -m exact_softmax_attention_03_b200.fit_exp2_poly
"""

from __future__ import annotations

import numpy as np


def fit(degree: int = 3, points: int = 4001):
    from scipy.optimize import linprog
    f = np.linspace(-0.5, 0.5, points)
    y = 2.0 ** f
    V = np.vstack([f ** k for k in range(degree + 1)]).T
    n = degree + 1
    c = np.zeros(n + 1)
    c[-1] = 1.0
    A = np.vstack([np.hstack([V, -y[:, None]]), np.hstack([-V, -y[:, None]])])
    b = np.concatenate([y, -y])
    res = linprog(c, A_ub=A, b_ub=b, bounds=[(None, None)] * n + [(0, None)], method="highs")
    return res.x[:n].astype(np.float32), float(res.x[-1])


if __name__ == "__main__":
    coef, err = fit()
    print("coefficients (c0..c3):", [float(x).hex() for x in coef])
    print("max relative error:", err)
