"""Provenance of the coefficients of exp2_poly2 (sm100.cuh): a minimax fit of
2^f on [-1/2, 1/2] for the smallest relative error, by linear programming
(minimise t subject to |p(f_i) - 2^f_i| <= t 2^f_i on a dense grid), then
rounded to fp32 and checked with fp32 Horner evaluation as the kernel runs it.

    python exp2_poly_fit.py        # prints degree 3 and 4 fits
"""
import numpy as np
from scipy.optimize import linprog


def fit(deg: int, points: int = 4001):
    """fp32 coefficients c0..c_deg and the LP's max relative error."""
    f = np.linspace(-0.5, 0.5, points)
    y = np.exp2(f)
    n = deg + 1
    V = np.vander(f, n, increasing=True)          # c0 + c1 f + ...
    A1 = np.hstack([V, -y[:, None]])
    A2 = np.hstack([-V, -y[:, None]])
    res = linprog(np.r_[np.zeros(n), 1.0], A_ub=np.vstack([A1, A2]), b_ub=np.r_[y, -y],
                  bounds=[(None, None)] * n + [(0, None)], method="highs")
    return res.x[:n].astype(np.float32), float(res.x[-1])


def horner_max_rel(c32) -> float:
    """Max relative error of fp32 Horner evaluation of c32 on [-1/2, 1/2]."""
    ff = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.full_like(ff, c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        p = (p * ff + c32[k]).astype(np.float32)
    return float(np.abs(p.astype(np.float64) / np.exp2(ff.astype(np.float64)) - 1).max())


if __name__ == "__main__":
    for deg in (3, 4):
        c32, lp = fit(deg)
        print(deg, [float(x) for x in c32], "lp max rel", lp, "fp32 horner max rel", horner_max_rel(c32))
