"""Coefficients of the cubic the forward kernel uses for part of its exponentials.

The kernel evaluates 2^x for x in [-124, 132] as 2^n * 2^f, with n = round(x) and
f = x - n in [-1/2, 1/2] (a Cody-Waite range reduction); 2^n goes into the
exponent field and 2^f = 1 + c1 f + c2 f^2 + c3 f^3.  The coefficients minimise
the largest relative error of the cubic over [-1/2, 1/2] with p(0) = 1 held
exactly; the minimax problem is a linear programme in (c1, c2, c3, t):

    minimise t  subject to  |(1 + c1 f + c2 f^2 + c3 f^3) / 2^f - 1| <= t

on a dense grid of f.  Run it to print the coefficients and the error bound;
fwd_kernel.cuh holds the printed values (as fp32).
"""
import numpy as np
from scipy.optimize import linprog


def fit(points=4001):
    f = np.linspace(-0.5, 0.5, points)
    w = np.exp2(-f)  # the relative error is (p(f) - 2^f) / 2^f = p(f) w - 1
    a = np.stack([f * w, f * f * w, f ** 3 * w], axis=1)
    ones = np.ones_like(f)
    # p w - 1 <= t  and  1 - p w <= t, with p w = w + a c
    a_ub = np.concatenate([np.hstack([a, -ones[:, None]]), np.hstack([-a, -ones[:, None]])])
    b_ub = np.concatenate([1 - w, w - 1])
    res = linprog(c=[0, 0, 0, 1], A_ub=a_ub, b_ub=b_ub, bounds=[(None, None)] * 3 + [(0, None)], method="highs")
    assert res.success
    return res.x[:3], res.x[3]


def max_rel_error(c, points=200001):
    f = np.linspace(-0.5, 0.5, points)
    c = np.float32(c).astype(np.float64)  # as the kernel holds them
    p = 1 + f * (c[0] + f * (c[1] + f * c[2]))
    return float(np.max(np.abs(p / np.exp2(f) - 1)))


if __name__ == "__main__":
    c, t = fit()
    print("c1, c2, c3 =", ", ".join(f"{float(np.float32(x))!r}f" for x in c))
    print(f"max relative error {t:.4e} (fp32 coefficients: {max_rel_error(c):.4e})")
