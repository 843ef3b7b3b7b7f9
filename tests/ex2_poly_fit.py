"""Remez fit of the polynomial behind the softmax's FMA-pipe exponential.

The kernel computes 2^x as 2^j * p(f), with j = round(x) and f = x - j in
[-1/2, 1/2], where p is the degree-3 polynomial of minimal maximum RELATIVE
error |p(f) - 2^f| / 2^f on that interval (all four coefficients free).  This
script finds p with the Remez exchange algorithm: solve for the coefficients
and the levelled error E on n + 2 = 5 reference points where the weighted
error alternates in sign, move the references to the extrema of the error
curve, repeat until they stop moving.  Run it to print the coefficients:

    python tests/ex2_poly_fit.py
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
HALF = 0.5


def _error(c, x):
    p = np.polynomial.polynomial.polyval(x, c)
    return (p - np.exp2(x)) / np.exp2(x)


def remez(degree: int = DEGREE, iters: int = 60, grid: int = 400001):
    """Coefficients c0..c_degree (lowest first) of the minimax-relative
    polynomial for 2^f on [-1/2, 1/2], and its maximum relative error."""
    n = degree + 2                                   # reference points
    ref = HALF * np.cos(np.linspace(np.pi, 0.0, n))  # Chebyshev start, ascending
    xs = np.linspace(-HALF, HALF, grid)
    c = None
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  ->  sum_k c_k x_i^k - (-1)^i E 2^x_i = 2^x_i
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(ref))
        c = sol[:degree + 1]
        err = _error(c, xs)
        # new references: the endpoints and the interior extrema of the error
        d = np.diff(err)
        interior = np.nonzero(d[:-1] * d[1:] < 0)[0] + 1
        idx = np.concatenate(([0], interior, [grid - 1]))
        if len(idx) != n:
            break
        new_ref = xs[idx]
        if np.allclose(new_ref, ref, atol=1e-12):
            ref = new_ref
            break
        ref = new_ref
    return c, float(np.abs(_error(c, xs)).max())


if __name__ == "__main__":
    coeffs, e = remez()
    print("coefficients (c0..c3):", [float(v) for v in coeffs])
    print("max relative error:", e)
