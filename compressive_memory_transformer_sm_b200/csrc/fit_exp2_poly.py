"""Fits the cubic used by exp2_poly() in sm100_attn.cuh.

2^x is evaluated as 2^n * p(f) with n = round(x) and f = x - n in
[-1/2, 1/2] (range reduction to the nearest integer, as in Cody and Waite's
scheme for exponentials).  p is the degree-3 polynomial minimising the maximum
relative error |p(f) / 2^f - 1| on a dense grid of [-1/2, 1/2], found as a
linear programme (discrete minimax).  Prints the coefficients c0..c3 (as
float32) and the error bound they achieve in float64 and after rounding the
coefficients to float32.
"""

import numpy as np
from scipy.optimize import linprog


def fit(degree=3, points=4001):
    f = np.linspace(-0.5, 0.5, points)
    t = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True)  # columns f^0 .. f^d
    # minimise e subject to  |V c - t| <= e t   (relative error)
    n = degree + 1
    cost = np.zeros(n + 1)
    cost[-1] = 1.0
    A = np.vstack([np.hstack([V, -t[:, None]]), np.hstack([-V, -t[:, None]])])
    b = np.concatenate([t, -t])
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * n + [(0, None)], method="highs")
    c = res.x[:n]
    c32 = c.astype(np.float32)
    fine = np.linspace(-0.5, 0.5, 200001)
    err64 = np.max(np.abs(np.polyval(c[::-1], fine) / np.exp2(fine) - 1))
    err32 = np.max(np.abs(np.polyval(c32.astype(np.float64)[::-1], fine) / np.exp2(fine) - 1))
    return c32, err64, err32


if __name__ == "__main__":
    c, e64, e32 = fit()
    for i, v in enumerate(c):
        print(f"c{i} = {float(v):.9e}f  (bits 0x{np.float32(v).view(np.uint32):08x})")
    print(f"max relative error: {e64:.3e} (exact coefficients), {e32:.3e} (float32 coefficients)")
