"""Fit the polynomial used by the forward kernel's software exp2.

Method: Cody & Waite range reduction (x = j + f, j = round(x), f in [-1/2, 1/2],
2^x = 2^j * 2^f) and a degree-3 polynomial p(f) ~ 2^f chosen by the Remez exchange
algorithm to minimise the maximum RELATIVE error on [-1/2, 1/2], with p(0) left
free.  Run it to print the coefficients that exp2_poly.cuh embeds:

    python context_zigzag_cp_b200/csrc/gen_exp2_poly.py
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez(degree: int = DEGREE, iters: int = 40):
    n = degree + 2
    # Chebyshev extrema as the initial reference set
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve sum_i c_i x^i + (-1)^j E 2^x = 2^x  (relative error equioscillation)
        f = np.exp2(x)
        A = np.zeros((n, n))
        for i in range(degree + 1):
            A[:, i] = x ** i
        A[:, -1] = ((-1.0) ** np.arange(n)) * f
        sol = np.linalg.solve(A, f)
        c = sol[:-1]
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        # new reference: extrema of the error, one per sign-alternating segment
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        cand = np.array(idx)
        # keep n alternating extrema with the largest magnitudes
        pts = []
        for i in cand:
            if pts and np.sign(err[i]) == np.sign(err[pts[-1]]):
                if abs(err[i]) > abs(err[pts[-1]]):
                    pts[-1] = i
            else:
                pts.append(i)
        while len(pts) > n:
            if abs(err[pts[0]]) < abs(err[pts[-1]]):
                pts.pop(0)
            else:
                pts.pop()
        if len(pts) < n:
            break
        x = grid[pts]
    c32 = c.astype(np.float32)
    err32 = np.abs(np.polyval(c32.astype(np.float64)[::-1], grid) / np.exp2(grid) - 1.0).max()
    return c32, float(err32)


if __name__ == "__main__":
    c, e = remez()
    for i, v in enumerate(c):
        print(f"c{i} = {float(v)!r}f  // {v.view(np.uint32):#010x}")
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}  (bf16 half-ulp = {2**-9:.3e})")
