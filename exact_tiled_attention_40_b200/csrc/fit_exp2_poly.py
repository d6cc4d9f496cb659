"""Fits the cubic used by the forward kernel's FMA-pipe exp2.

Method: Cody-Waite style range reduction 2^x = 2^n * 2^f with n = round(x) and
f in [-1/2, 1/2], then a cubic p(f) ~ 2^f chosen to minimise the maximum
relative error on [-1/2, 1/2] (Remez exchange on the relative error, started
from Chebyshev nodes).  Prints the coefficients c0..c3 (p = c0 + c1 f + c2 f^2
+ c3 f^3) as float32 literals and the achieved maximum relative error.
"""
import numpy as np


def remez_rel(deg=3, a=-0.5, b=0.5, iters=30):
    f = lambda x: np.exp2(x)
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new extrema: sign changes partition
        idx = [0]
        s = np.sign(err)
        for i in range(1, len(grid)):
            if s[i] != s[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) < n:
            break
        # keep n alternating extrema with the largest magnitude
        while len(idx) > n:
            j = int(np.argmin([abs(err[i]) for i in idx]))
            idx.pop(j)
        x = grid[idx]
    return c, np.max(np.abs(err))


if __name__ == "__main__":
    c, e = remez_rel()
    c32 = c.astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.float32(c32[3])
    for k in (2, 1, 0):
        p = (p * grid + c32[k]).astype(np.float32)
    rel32 = np.max(np.abs(p.astype(np.float64) - np.exp2(grid.astype(np.float64)))
                   / np.exp2(grid.astype(np.float64)))
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v).hex()}  # {float(v):.9g}")
    print(f"max relative error: {e:.3e} (float64 coefficients), {rel32:.3e} (float32 Horner)")
