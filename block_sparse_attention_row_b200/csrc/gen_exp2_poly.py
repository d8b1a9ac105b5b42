"""Derives the coefficients of the software 2^f used by the attention kernel.

Method: Cody-Waite style range reduction (x = n + f, n = round(x), f in
[-1/2, 1/2], 2^x = 2^n * 2^f) and a degree-3 polynomial for 2^f on
[-1/2, 1/2] chosen by the Remez exchange algorithm to minimise the maximum
relative error. Run it to print the constants written in sa_attn_kernel.cuh.
"""
import numpy as np


def remez_relative(deg=3, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)
    n = deg + 2
    # start from Chebyshev extrema
    k = np.arange(n)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative error alternation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        grid = np.linspace(lo, hi, 200001)
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new extrema: one per sign-alternating segment
        sgn = np.sign(err)
        idx = np.nonzero(np.diff(sgn))[0]
        bounds = np.concatenate(([0], idx + 1, [len(grid)]))
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(ext) != n:
            break
        x = grid[ext]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez_relative()
    c32 = c.astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 100001)
    err32 = np.max(np.abs((np.polyval(c32[::-1].astype(np.float64), grid) - np.exp2(grid)) / np.exp2(grid)))
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v):.9e}f  ({float(v).hex()})")
    print(f"max relative error: {e:.3e} (fp64 coefficients), {err32:.3e} (fp32 coefficients)")
