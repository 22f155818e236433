"""Derivation of the FMA-pipe 2^x polynomial of the attention kernel.

The kernel splits x = n + f with n = round(x) and f in [-1/2, 1/2], evaluates 2^f with a
cubic c3 f^3 + c2 f^2 + c1 f + c0 in Horner form, and adds n to the exponent field.  The
cubic minimises the maximum *relative* error |p(f) / 2^f - 1| over [-1/2, 1/2] (a relative
bound is what survives the exponent add).  It is found with Lawson's algorithm: weighted
least squares whose weights are multiplied, after each solve, by the absolute error at each
point and renormalised; the weights concentrate on the equioscillation points and the
solution tends to the minimax one.

    python tests/golden/fit_exp2_poly.py     # prints the coefficients and the max error

Only numpy; nothing here is imported by the library or by the oracle.
"""
from __future__ import annotations

import numpy as np


def lawson_fit(degree: int = 3, n_points: int = 4001, iters: int = 400):
    f = np.linspace(-0.5, 0.5, n_points)
    g = np.exp2(f)
    # relative error e = p(f)/g - 1 is linear in the coefficients: A c - 1 with A[i,k] = f_i^k / g_i
    A = np.stack([f ** k / g for k in range(degree + 1)], axis=1)
    w = np.full(n_points, 1.0 / n_points)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], sw, rcond=None)
        e = np.abs(A @ c - 1.0)
        w = w * e
        w /= w.sum()
    return c, float(np.max(np.abs(A @ c - 1.0)))


if __name__ == "__main__":
    c, err = lawson_fit()
    print("c0..c3 =", ", ".join(f"{x:.8f}" for x in c))
    print(f"max relative error on [-1/2, 1/2]: {err:.3e}")
