"""Coefficients of the polynomial 2^f ~ c0 + c1 f + ... + cd f^d on [-1/2, 1/2]
used by the kernels' FMA-pipe exp2 (csrc/sm100.cuh, exp2_poly).

Method: Cody & Waite argument reduction (2^y = 2^n * 2^f, n = round(y),
f = y - n in [-1/2, 1/2]) followed by a minimax polynomial for 2^f in the
relative-error sense, computed with the Remez exchange algorithm (Remez 1934).
Coefficients are rounded to f32 and the final error is re-measured in f32
Horner arithmetic. Run: python gen_exp2_poly.py [degree]
"""
import sys

import numpy as np


def remez_rel(deg, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)
    n = deg + 2
    # Chebyshev extrema as the initial reference
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    c = None
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i) for c_0..c_deg, E
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c, E = sol[:deg + 1], sol[deg + 1]
        grid = np.linspace(lo, hi, 200001)
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        idx = [0]
        sgn = np.sign(err)
        segs = np.split(np.arange(len(grid)), np.where(np.diff(sgn) != 0)[0] + 1)
        ext = [s[np.argmax(np.abs(err[s]))] for s in segs]
        if len(ext) >= n:
            # keep the n largest alternating extrema
            while len(ext) > n:
                k = np.argmin([abs(err[e]) for e in ext])
                ext.pop(k if k in (0, len(ext) - 1) else k)
            x = grid[ext]
    return c


def f32_horner_err(c):
    c32 = np.asarray(c, dtype=np.float32)
    g = np.linspace(-0.5, 0.5, 2000001).astype(np.float32)
    acc = np.full_like(g, c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        acc = (acc * g + c32[k]).astype(np.float32)
    ref = np.exp2(g.astype(np.float64))
    return float(np.max(np.abs(acc.astype(np.float64) - ref) / ref)), c32


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c = remez_rel(deg)
    err, c32 = f32_horner_err(c)
    print(f"degree {deg}: max relative error {err:.3e} (f32 Horner)")
    for k, v in enumerate(c32):
        print(f"  c{k} = {float(v):.9e}f  ({v.view(np.uint32):#010x})")
