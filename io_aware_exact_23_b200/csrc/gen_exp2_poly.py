"""Fit the cubic used by the kernels' software exp2: p(f) ~ 2^f on f in [-1/2, 1/2].

Method: Remez exchange for the minimax *relative* error of a degree-3
polynomial (weight 1/2^f), starting from Chebyshev extrema.  The kernels
evaluate 2^x = 2^n * p(x - n) with n = rint(x), adding n to p's exponent field;
this script prints the coefficients that fa_fwd.cuh hard-codes and the error
bound they achieve.  Run: ``python gen_exp2_poly.py``.
"""
from __future__ import annotations

import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def fit(deg=DEG, iters=30):
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k / (n - 1))[::-1]
    f = lambda t: np.exp2(t)  # noqa: E731
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E f(x_i) = f(x_i)   (relative-error equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        grid = np.linspace(LO, HI, 200001)
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: alternating extrema of err
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        cand = grid[idx]
        ev = err[idx]
        # keep n points with alternating signs and largest magnitudes
        pts, vals = [cand[0]], [ev[0]]
        for t, v in zip(cand[1:], ev[1:]):
            if np.sign(v) == np.sign(vals[-1]):
                if abs(v) > abs(vals[-1]):
                    pts[-1], vals[-1] = t, v
            else:
                pts.append(t)
                vals.append(v)
        while len(pts) > n:
            if abs(vals[0]) < abs(vals[-1]):
                pts.pop(0)
                vals.pop(0)
            else:
                pts.pop()
                vals.pop()
        if len(pts) == n:
            x = np.array(pts)
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = fit()
    c32 = np.array(c, dtype=np.float32)
    grid = np.linspace(LO, HI, 200001)
    p32 = np.zeros_like(grid, dtype=np.float32)
    for ci in c32[::-1]:
        p32 = p32 * grid.astype(np.float32) + ci
    e32 = float(np.abs((p32.astype(np.float64) - np.exp2(grid)) / np.exp2(grid)).max())
    for i, ci in enumerate(c32):
        print(f"c{i} = {float(ci)!r}f")
    print(f"max relative error: {e:.3e} (fp64 coefficients), {e32:.3e} (fp32 Horner)")
