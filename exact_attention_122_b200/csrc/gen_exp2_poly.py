"""Fit the polynomial used by the kernel's software 2^x.

Method: Cody-Waite range reduction x = n + f with n = rint(x), f in
[-1/2, 1/2], so 2^x = 2^n * 2^f; 2^f is approximated by a degree-3
polynomial whose coefficients minimise the maximum relative error on
[-1/2, 1/2] (Remez exchange on the relative error, started from Chebyshev
nodes).  Run it to reproduce the constants in fa_fwd_sm100.cu:

    python exact_attention_122_b200/csrc/gen_exp2_poly.py
"""

import numpy as np


def remez_relative(deg=3, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)
    # initial reference: Chebyshev extrema
    k = np.arange(deg + 2)
    xs = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k / (deg + 1))[::-1]
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (equioscillating relative error)
        A = np.zeros((deg + 2, deg + 2))
        for i, x in enumerate(xs):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x)
        sol = np.linalg.solve(A, f(xs))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        idx = [0]
        sgn = np.sign(err)
        for j in range(1, len(grid)):
            if sgn[j] != sgn[idx[-1]]:
                idx.append(j)
            elif abs(err[j]) > abs(err[idx[-1]]):
                idx[-1] = j
        if len(idx) < deg + 2:
            break
        # keep deg+2 points with the largest errors, alternating
        while len(idx) > deg + 2:
            if abs(err[idx[0]]) < abs(err[idx[-1]]):
                idx.pop(0)
            else:
                idx.pop()
        xs = grid[idx]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez_relative()
    c32 = c.astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = ((c32[3] * grid + c32[2]) * grid + c32[1]) * grid + c32[0]
    e32 = np.max(np.abs(p.astype(np.float64) / np.exp2(grid.astype(np.float64)) - 1))
    for i, ci in enumerate(c32):
        print(f"C{i} = {float(ci):.9e}f  ({float(ci).hex()})")
    print(f"max relative error: {e:.3e} (float64 coefficients), {e32:.3e} (float32 Horner)")
