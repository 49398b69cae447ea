"""Fits the polynomial the kernel uses for 2^f on f in [-1/2, 1/2].

Method: minimax (smallest maximum relative error) polynomial of degree 3,
found as a linear program over a dense grid: minimise e subject to
|p(f_i) / 2^f_i - 1| <= e for all grid points f_i (the discrete Chebyshev
approximation problem). The coefficients are then rounded to float32 and the
error re-measured by evaluating the rounded polynomial with Horner's rule in
float32, as the kernel does.

    python gen_exp2_poly.py          # prints the coefficients and the error
"""

import numpy as np
from scipy.optimize import linprog

DEGREE = 3


def fit(degree: int = DEGREE, n: int = 4001):
    f = np.linspace(-0.5, 0.5, n)
    target = np.exp2(f)
    # variables: c_0..c_degree, e; minimise e
    V = np.vander(f, degree + 1, increasing=True) / target[:, None]  # p(f)/2^f
    ones = np.ones((n, 1))
    A = np.vstack([np.hstack([V, -ones]), np.hstack([-V, -ones])])
    b = np.concatenate([np.ones(n), -np.ones(n)])
    c = np.zeros(degree + 2)
    c[-1] = 1.0
    res = linprog(c, A_ub=A, b_ub=b, bounds=[(None, None)] * (degree + 1) + [(0, None)],
                  method="highs")
    assert res.success, res.message
    return res.x[:-1], res.x[-1]


def max_rel_error_f32(coeffs, n: int = 200001):
    c = np.asarray(coeffs, dtype=np.float32)
    f = np.linspace(-0.5, 0.5, n).astype(np.float32)
    p = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + c[k]).astype(np.float32)   # float32 Horner, as on the device
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    coeffs, e = fit()
    c32 = np.asarray(coeffs, dtype=np.float32)
    print("degree", DEGREE, "minimax relative error (float64 coefficients):", e)
    print("max relative error, float32 coefficients and Horner:", max_rel_error_f32(c32))
    for k, v in enumerate(c32):
        print(f"  c{k} = {float(v)!r}f   // {v.view(np.uint32):#010x}")
