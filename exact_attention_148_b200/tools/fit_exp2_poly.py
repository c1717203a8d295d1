"""Fit the polynomial used by the prefill kernel's FMA-pipe exp2.

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]
(Cody & Waite's argument reduction, "Software Manual for the Elementary
Functions", 1980); 2^n is applied by adding n to the float's exponent field,
and 2^f comes from a polynomial p(f).  This script finds the degree-3
polynomial that minimises the maximum *relative* error on [-1/2, 1/2] with the
Remez exchange algorithm (p(0) is left free: the fit is minimax over the
interval).

Run: python -m exact_attention_148_b200.tools.fit_exp2_poly
Prints the coefficients (c0 + c1 f + c2 f^2 + c3 f^3) and the error bound.
"""
import numpy as np


def remez_rel(deg=3, iters=40, a=-0.5, b=0.5):
    n = deg + 2
    # initial reference: Chebyshev extrema mapped to [a, b]
    xs = 0.5 * (a + b) - 0.5 * (b - a) * np.cos(np.pi * np.arange(n) / (n - 1))
    grid = np.linspace(a, b, 200001)
    target = np.exp2(grid)
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E * 2^{x_i} = 2^{x_i}
        A = np.zeros((n, n))
        for i, x in enumerate(xs):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(xs))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - target) / target
        # new reference: extrema of the error curve, one per sign run
        s = np.sign(err)
        idx = []
        start = 0
        for k in range(1, len(grid) + 1):
            if k == len(grid) or s[k] != s[start]:
                seg = np.arange(start, k)
                idx.append(seg[np.argmax(np.abs(err[seg]))])
                start = k
        if len(idx) >= n:
            # keep the n alternating extrema with the largest errors
            while len(idx) > n:
                drop = 0 if abs(err[idx[0]]) < abs(err[idx[-1]]) else len(idx) - 1
                idx.pop(drop)
            xs = grid[idx]
    return c, np.max(np.abs(err))


if __name__ == "__main__":
    c, e = remez_rel()
    print("coefficients c0..c3:", ", ".join(f"{x:.9g}" for x in c))
    print("max relative error on [-1/2,1/2]:", e)
    f = np.linspace(-0.5, 0.5, 100001, dtype=np.float32)
    c32 = c.astype(np.float32)
    p = ((c32[3] * f + c32[2]) * f + c32[1]) * f + c32[0]
    print("float32 evaluation max rel error:", np.max(np.abs(p / np.exp2(f.astype(np.float64)) - 1)))
