"""Fit of the polynomial behind the query-tile kernel's FMA-pipe exp2.

The kernel computes a share of its exponentials 2^x without the
special-function unit, by Cody-Waite range reduction: x = j + f with
j = rint(x) and f in [-1/2, 1/2], 2^x = 2^j * 2^f, where 2^j is placed into
the float's exponent field with an integer add and 2^f comes from a
polynomial p(f). This script finds the p of a given degree that minimises
the largest relative error |p(f) / 2^f - 1| on [-1/2, 1/2] (the Remez
exchange algorithm on the relative error), rounds its coefficients to
float32, and reports the error of the rounded polynomial on a dense grid.

    python ragged_paged_kv_b200/csrc/exp2_poly_fit.py [degree]

The printed coefficients are the ones attn_tc.cu uses (degree 4).
"""
import sys

import numpy as np


def remez_relative(deg, lo=-0.5, hi=0.5, iters=30):
    n = deg + 2
    # start from Chebyshev extrema
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i for the coefficients and E
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extrema of the error between its sign changes
        idx = []
        sign = np.sign(err)
        start = 0
        for k in range(1, len(grid) + 1):
            if k == len(grid) or sign[k] != sign[start]:
                seg = np.arange(start, k)
                idx.append(seg[np.argmax(np.abs(err[seg]))])
                start = k
        idx = np.array(idx)
        if len(idx) > n:  # keep the n largest alternating extrema
            while len(idx) > n:
                drop = 0 if abs(err[idx[0]]) < abs(err[idx[-1]]) else len(idx) - 1
                idx = np.delete(idx, drop)
        if len(idx) == n:
            x = grid[idx]
    return c


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c = remez_relative(deg)
    c32 = c.astype(np.float32)
    f = np.linspace(-0.5, 0.5, 2000001)
    p = np.zeros_like(f, dtype=np.float64)
    for ci in c32[::-1].astype(np.float64):
        p = p * f + ci
    rel = np.abs(p / 2.0 ** f - 1.0).max()
    print(f"degree {deg}: max relative error of the float32-rounded polynomial {rel:.3e} (2^{np.log2(rel):.2f})")
    for i, ci in enumerate(c32):
        print(f"  c{i} = {float(ci)!r:>24}  ({float(ci).hex()})")


if __name__ == "__main__":
    main()
