"""Minimax polynomial for 2^f on [-1/2, 1/2] (relative error), used by the
forward kernel to evaluate part of its exponentials on the FMA pipe.

Method: Remez exchange (E. Ya. Remez, 1934) on the weighted error
e(f) = p(f) / 2^f - 1 over [-1/2, 1/2], starting from Chebyshev nodes.  The
kernel reduces x to n + f with n = round(x) (adding and subtracting
1.5 * 2^23 in fp32, which rounds to nearest) and scales p(f) by 2^n by adding
n to the exponent field.  Running this module prints the coefficients that
fm_common.cuh holds; tests/test_exp2_poly.py re-derives them and checks the
error bound of the fp32 evaluation.
"""
from __future__ import annotations

import numpy as np


def remez_exp2(degree: int, iters: int = 30, grid: int = 20001):
    a, b = -0.5, 0.5
    n = degree + 2
    k = np.arange(n)
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * (n - 1 - k) / (n - 1))  # Chebyshev extrema
    fine = np.linspace(a, b, grid)
    coef = None
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i   (relative-error equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1.0) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        coef = sol[:degree + 1]
        err = np.polyval(coef[::-1], fine) / 2.0 ** fine - 1.0
        # new reference: extremum of each sign run
        sign = np.sign(err)
        idx, start = [], 0
        for t in range(1, grid + 1):
            if t == grid or sign[t] != sign[start]:
                seg = np.arange(start, t)
                idx.append(seg[np.argmax(np.abs(err[seg]))])
                start = t
        if len(idx) < n:
            break
        # keep the n extrema with the largest error that alternate
        idx = np.array(idx)
        while len(idx) > n:
            drop = 0 if abs(err[idx[0]]) < abs(err[idx[-1]]) else len(idx) - 1
            idx = np.delete(idx, drop)
        x = fine[idx]
    err = np.polyval(coef[::-1], fine) / 2.0 ** fine - 1.0
    return coef, float(np.max(np.abs(err)))


def as_f32(coef):
    return [float(np.float32(c)) for c in coef]


if __name__ == "__main__":
    for deg in (2, 3, 4):
        c, e = remez_exp2(deg)
        print(f"degree {deg}: max rel error {e:.3e}")
        print("  coefficients (c0..c%d): %s" % (deg, ", ".join(f"{v:.9e}f" for v in as_f32(c))))
