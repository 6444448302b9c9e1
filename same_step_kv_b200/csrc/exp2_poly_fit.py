"""Fits the cubic that attn_kernel uses for part of its exponentials.

2^x = 2^n * 2^f with n = round(x), f = x - n in [-1/2, 1/2] (range reduction
in the manner of Cody and Waite); 2^f is approximated by the degree-3
polynomial with the smallest maximum relative error on [-1/2, 1/2], found by
the Remez exchange algorithm.  The coefficients are then rounded to float32
and the error re-measured.  Run:  python exp2_poly_fit.py
"""
import numpy as np


def remez_relative(deg=3, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)
    # start from Chebyshev extrema
    k = np.arange(deg + 2)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k / (deg + 1))[::-1]
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative error equioscillation)
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(xi)
        c = np.linalg.solve(A, f(x))
        coef = c[:deg + 1]
        err = (np.polyval(coef[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        s = np.sign(err)
        idx = np.nonzero(np.diff(s))[0]
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(ext) != deg + 2:
            break
        x = grid[ext]
    return coef, np.max(np.abs(err))


if __name__ == "__main__":
    coef, e64 = remez_relative()
    c32 = coef.astype(np.float32)
    g = np.linspace(-0.5, 0.5, 400001)
    p = np.float32(c32[3])
    for c in c32[2::-1]:
        p = (p * g.astype(np.float32) + c).astype(np.float32)
    e32 = np.max(np.abs(p.astype(np.float64) - np.exp2(g)) / np.exp2(g))
    print("max relative error: fp64 coefficients %.3e, float32 Horner %.3e" % (e64, e32))
    for i, c in enumerate(c32):
        print("c%d = %.9ef" % (i, c))
