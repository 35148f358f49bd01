"""Fit the polynomial behind the kernels' software exp2 (build-time helper).

Method: Cody-Waite style range reduction, 2^x = 2^n * 2^f with n = rint(x) and
f = x - n in [-1/2, 1/2], then a polynomial p(f) ~ 2^f of degree 3 that
minimises the maximum relative error on a dense grid (discrete minimax,
solved as a linear programme). Prints the coefficients in float32 and the
maximum relative error of the float32 Horner evaluation.

    python exact_io_aware_96_b200/csrc/fit_exp2_poly.py
"""
import numpy as np
from scipy.optimize import linprog


def fit(degree=3, n=4001):
    f = np.linspace(-0.5, 0.5, n)
    y = np.exp2(f)
    V = np.vander(f, degree + 1, increasing=True) / y[:, None]   # relative residual rows
    # variables: c_0..c_d, e ; minimise e s.t. |V c - 1| <= e
    ncoef = degree + 1
    cost = np.zeros(ncoef + 1)
    cost[-1] = 1.0
    A = np.vstack([np.hstack([V, -np.ones((n, 1))]), np.hstack([-V, -np.ones((n, 1))])])
    b = np.concatenate([np.ones(n), -np.ones(n)])
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * (ncoef + 1), method="highs")
    return res.x[:ncoef]


def horner32(c, f):
    c = [np.float32(x) for x in c]
    f = np.float32(f) if np.isscalar(f) else f.astype(np.float32)
    p = c[-1]
    for ci in reversed(c[:-1]):
        p = np.float32(p * f + ci)
    return p


if __name__ == "__main__":
    c = fit()
    c32 = [float(np.float32(x)) for x in c]
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    err = np.max(np.abs(horner32(c32, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1))
    print("coefficients (c0..c3):", ", ".join(f"{x:.9g}f" for x in c32))
    print(f"max relative error on [-1/2, 1/2]: {err:.3e}")
