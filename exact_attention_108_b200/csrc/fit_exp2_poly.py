"""Fits the coefficients of the degree-3 polynomial p(f) ~ 2^f, f in [-1/2, 1/2],
used by exp2_poly_x2 in sm100.cuh: minimise the maximum relative error
|p(f) / 2^f - 1| on a dense grid (a linear program), with p(0) = 1 held exact.

    python exact_attention_108_b200/csrc/fit_exp2_poly.py
"""
import numpy as np
from scipy.optimize import linprog


def fit(deg: int = 3, points: int = 4001):
    f = np.linspace(-0.5, 0.5, points)
    y = np.exp2(f)
    a_ub, b_ub = [], []
    for fi, yi in zip(f, y):
        row = [fi ** k for k in range(1, deg + 1)]
        a_ub.append(row + [-yi])               # p - y <= t y
        b_ub.append(yi - 1.0)
        a_ub.append([-r for r in row] + [-yi])  # y - p <= t y
        b_ub.append(1.0 - yi)
    res = linprog([0.0] * deg + [1.0], A_ub=np.array(a_ub), b_ub=np.array(b_ub),
                  bounds=[(None, None)] * deg + [(0, None)], method="highs")
    coef = np.concatenate([[1.0], res.x[:deg]]).astype(np.float32)
    ff = f.astype(np.float32)
    p = np.float32(coef[-1])
    for k in range(deg - 1, -1, -1):
        p = (p * ff + coef[k]).astype(np.float32)
    return coef, float(np.max(np.abs(p.astype(np.float64) / y - 1.0)))


if __name__ == "__main__":
    coef, err = fit()
    print("coefficients c0..c3:", [repr(float(c)) for c in coef])
    print("max relative error (fp32 Horner): %.3e" % err)
