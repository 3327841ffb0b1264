"""Coefficients of the cubic that the attention kernel uses for 2^f on the FMA pipe.

    python free_clustered_block_b200/csrc/exp2_poly_fit.py

The attention kernel evaluates part of its exponentials 2^t without the MUFU
ex2 unit: t = n + f with n = round(t) and f in [-1/2, 1/2], 2^f by a cubic
p(f), and n added into the exponent field. This script finds p by the Remez
exchange algorithm (E. Ya. Remez, 1934; e.g. Cheney, "Introduction to
Approximation Theory", ch. 3) for the least maximum RELATIVE error
max |p(f) / 2^f - 1| over [-1/2, 1/2], then rounds the coefficients to fp32
and reports the error of the rounded cubic on a dense grid. The printed
constants are the ones in attend_tc.cu (exp2_poly2).
"""
from __future__ import annotations

import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def _solve(ref):
    # p(x_i) - 2^x_i = (-1)^i E 2^x_i  ->  sum_k c_k x_i^k - (-1)^i 2^x_i E = 2^x_i
    n = len(ref)
    A = np.zeros((n, DEG + 2))
    for i, x in enumerate(ref):
        A[i, :DEG + 1] = [x ** k for k in range(DEG + 1)]
        A[i, DEG + 1] = -((-1) ** i) * 2.0 ** x
    sol = np.linalg.solve(A, 2.0 ** ref)
    return sol[:DEG + 1], sol[DEG + 1]


def rel_err(coef, x):
    p = np.polyval(coef[::-1], x)
    return p / 2.0 ** x - 1.0


def remez(iters=30):
    # Chebyshev nodes as the first reference
    k = np.arange(DEG + 2)
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (DEG + 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        coef, E = _solve(ref)
        e = rel_err(coef, grid)
        # new reference: the extremum of each sign run of the error, end points included
        idx = [0]
        for i in range(1, grid.size - 1):
            if (e[i] - e[i - 1]) * (e[i + 1] - e[i]) <= 0:
                idx.append(i)
        idx.append(grid.size - 1)
        idx = np.array(sorted(set(idx)))
        # keep alternating extrema of largest magnitude
        alt = []
        for i in idx:
            if alt and np.sign(e[i]) == np.sign(e[alt[-1]]):
                if abs(e[i]) > abs(e[alt[-1]]):
                    alt[-1] = i
            else:
                alt.append(i)
        while len(alt) > DEG + 2:
            if abs(e[alt[0]]) < abs(e[alt[-1]]):
                alt.pop(0)
            else:
                alt.pop()
        if len(alt) < DEG + 2:
            break
        ref = grid[alt]
    return coef, abs(E)


def main():
    coef, E = remez()
    c32 = np.array(coef, dtype=np.float32)
    grid = np.linspace(LO, HI, 2000001)
    err32 = np.abs(rel_err(c32.astype(np.float64), grid)).max()
    print(f"levelled relative error (fp64 coefficients): {E:.3e}")
    print(f"max relative error with fp32 coefficients:   {err32:.3e}")
    for i, c in enumerate(c32):
        print(f"c{i} = {float(c):.10e}f  ({np.float32(c).view(np.uint32):#010x})")


if __name__ == "__main__":
    main()
