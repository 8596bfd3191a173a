"""Coefficients of the FMA-pipe exp2 used by the attention softmax.

2^x is split as 2^n * 2^f with n = rint(x) and f = x - n in [-1/2, 1/2]
(Cody & Waite's argument reduction); 2^f is a cubic whose coefficients
minimise the maximum relative error on [-1/2, 1/2], found by the Remez
exchange algorithm below. The softmax rounds P to bf16 (relative step
2^-8), so a relative error near 1e-4 is far below what the output can
show. Run: python fit_exp2_poly.py
"""
import numpy as np


def remez_relative(degree=3, lo=-0.5, hi=0.5, iters=30):
    f = lambda x: np.exp2(x)
    n = degree + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    ref = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # p(x_i) - f(x_i) = (-1)^i E f(x_i): linear in (c_0..c_d, E)
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, -1] = -((-1) ** i) * f(x)
        sol = np.linalg.solve(A, f(ref))
        c = sol[:-1]
        err = np.polyval(c[::-1], grid) / f(grid) - 1
        # new reference: the extrema of the error, one per sign-alternating run
        sign = np.sign(err)
        idx = [0]
        cur = 0
        for i in range(1, len(grid)):
            if sign[i] != sign[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        idx = np.array(idx)
        if len(idx) >= n:
            # keep the n largest consecutive alternating extrema
            best = max(range(len(idx) - n + 1), key=lambda s: np.min(np.abs(err[idx[s:s + n]])))
            ref = grid[idx[best:best + n]]
    return c, np.max(np.abs(err))


if __name__ == "__main__":
    c, e = remez_relative()
    c32 = c.astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 200001)
    e32 = np.max(np.abs(np.polyval(c32[::-1].astype(np.float64), grid) / np.exp2(grid) - 1))
    print("coefficients c0..c3 (fp32):", [float(x) for x in c32])
    print(f"max relative error: {e:.3e} (fp64 coefficients), {e32:.3e} (fp32 coefficients)")
