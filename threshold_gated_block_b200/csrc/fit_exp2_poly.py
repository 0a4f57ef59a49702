"""Fit the polynomial the softmax kernel uses for part of its exp2 evaluations.

The kernel evaluates 2^x for x <= 8 as 2^i * p(f), where i = round(x) and
f = x - i lies in [-1/2, 1/2]. p is the degree-3 polynomial that minimises the
maximum relative error |p(f) / 2^f - 1| on that interval, found here with the
Remez exchange algorithm (alternation theorem: the optimum equioscillates at
degree + 2 points). The exponent 2^i is applied by adding i to the float's
exponent field, so the relative error of the result is that of p.

Run: python fit_exp2_poly.py   (prints the coefficients and the error bound)
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez(degree: int = DEGREE, iters: int = 50):
    n = degree + 2
    # Chebyshev extrema as the starting reference
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    f = lambda t: np.exp2(t)
    for _ in range(iters):
        # Solve p(x_k) - f(x_k) = (-1)^k E f(x_k) for the coefficients and E (relative error).
        A = np.zeros((n, n))
        for r in range(n):
            A[r, :degree + 1] = x[r] ** np.arange(degree + 1)
            A[r, degree + 1] = -((-1) ** r) * f(x[r])
        sol = np.linalg.solve(A, f(x))
        c = sol[:degree + 1]
        err = np.polyval(c[::-1], grid) / f(grid) - 1.0
        # New reference: the extrema of the error between its sign changes.
        sign_change = np.nonzero(np.diff(np.sign(err)))[0]
        bounds = np.concatenate(([0], sign_change + 1, [len(grid)]))
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:]) if b1 > b0]
        if len(ext) < n:
            break
        ext = np.array(ext)
        if len(ext) > n:   # keep the n largest alternating extrema
            ext = ext[np.argsort(-np.abs(err[ext]))[:n]]
            ext.sort()
        x = grid[ext]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez()
    for i, ci in enumerate(c):
        print(f"c{i} = {np.float32(ci)!r}  ({ci:.10e})")
    print(f"max relative error on [{LO}, {HI}]: {e:.3e}")
