"""Fits the polynomial the kernel uses to compute 2^f on the FMA pipe.

Method: Cody-Waite style range reduction (x = n + f, n = round(x), |f| <= 1/2,
2^x = 2^n * 2^f with 2^n added into the exponent field) and a minimax
polynomial for 2^f on [-1/2, 1/2] in the relative-error sense, found with the
Remez exchange algorithm (E. Remez, 1934). Prints the coefficients
c0..cN of p(f) = c0 + c1 f + ... + cN f^N and the max relative error.

Run: python gen_exp2_poly.py [degree]
"""
import sys

import numpy as np


def remez_relative(degree, a=-0.5, b=0.5, iters=30):
    f = lambda x: np.exp2(x)
    n = degree
    # initial reference: Chebyshev extrema
    k = np.arange(n + 2)
    ref = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k[::-1] / (n + 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)
        A = np.zeros((n + 2, n + 2))
        for i, x in enumerate(ref):
            A[i, :n + 1] = x ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * f(x)
        sol = np.linalg.solve(A, f(ref))
        c = sol[:n + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        sign = np.sign(err)
        idx = [0]
        for i in range(1, len(grid)):
            if sign[i] != sign[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) >= n + 2:
            best = None
            for s in range(len(idx) - (n + 2) + 1):
                cand = idx[s:s + n + 2]
                m = min(abs(err[j]) for j in cand)
                if best is None or m > best[0]:
                    best = (m, cand)
            ref = grid[best[1]]
    err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_relative(deg)
    for i, ci in enumerate(c):
        print(f"c{i} = {np.float32(ci)!r}  # {ci:.17g}")
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
