"""Fit the polynomial the bf16 attention kernel uses to compute part of its exp2 values on the
FMA pipe instead of the MUFU unit.

Method: Cody-Waite style range reduction, 2^x = 2^j * 2^f with j = round(x) and f = x - j in
[-1/2, 1/2], and a degree-3 polynomial for 2^f whose maximum RELATIVE error on [-1/2, 1/2] is
minimised by the Remez exchange algorithm (equioscillation on 5 points). Run this script to
reproduce the coefficients printed into fwd_bf16_sm100.cu:

    python scaled_dot_product_16_b200/csrc/fit_exp2_poly.py
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    # start from Chebyshev extrema
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k / (n - 1))[::-1]
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  (relative error equioscillation)
        A = np.zeros((n, n))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: extrema of the error between sign changes
        sgn = np.sign(err)
        idx = np.concatenate([[0], np.nonzero(np.diff(sgn))[0] + 1, [len(grid)]])
        ext = [seg_start + np.argmax(np.abs(err[seg_start:seg_end]))
               for seg_start, seg_end in zip(idx[:-1], idx[1:])]
        if len(ext) != n:
            break
        x = grid[ext]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez()
    c32 = c.astype(np.float32)
    grid = np.linspace(LO, HI, 200001).astype(np.float32)
    # Horner in float32 as the kernel evaluates it
    p = np.float32(c32[3])
    p = p * grid + c32[2]
    p = p * grid + c32[1]
    p = p * grid + c32[0]
    e32 = float(np.max(np.abs(p.astype(np.float64) / 2.0 ** grid.astype(np.float64) - 1)))
    for i, ci in enumerate(c32):
        print(f"c{i} = {float(ci):.9e}f")
    print(f"max relative error: {e:.3e} (exact arithmetic), {e32:.3e} (float32 Horner)")
