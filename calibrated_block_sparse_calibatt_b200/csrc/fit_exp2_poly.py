"""Derives the coefficients of the FMA-pipe exp2 used by the tensor-core softmax.

Method (Cody and Waite's argument reduction, then a polynomial on the reduced
argument): 2^x = 2^n * 2^f with n an integer near x and f = x - n small.  2^f is
approximated by a cubic c0 + c1 f + c2 f^2 + c3 f^3 chosen to minimise the
maximum relative error on the reduced interval (Remez exchange, equioscillation
of the relative error on 5 points), here computed with numpy from scratch.  The
kernel rounds to nearest (n = rint(x), f in [-1/2, 1/2]) using the float
addition of 1.5 * 2^23, so no float-to-integer conversion instruction is used.  The
result only feeds bf16 attention probabilities (8-bit mantissa), so a relative
error near 1e-4 is far below their rounding step.

Run: python fit_exp2_poly.py  -> prints the coefficients and the error bound.
"""

import numpy as np


def remez_relative(degree=3, iters=30, lo=-0.5, hi=0.5):
    # initial reference: Chebyshev extrema mapped to [0, 1]
    m = degree + 2
    xs = lo + (hi - lo) * (0.5 - 0.5 * np.cos(np.pi * np.arange(m) / (m - 1)))
    for _ in range(iters):
        # solve sum c_k x^k - 2^x = (-1)^i E 2^x  (relative error equioscillates)
        a = np.zeros((m, m))
        for i, x in enumerate(xs):
            a[i, :degree + 1] = x ** np.arange(degree + 1)
            a[i, degree + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(a, 2.0 ** xs)
        c = sol[:degree + 1]
        grid = np.linspace(lo, hi, 200001)
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: extrema of the error on each sign-alternating segment
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = sorted(idx, key=lambda i: -abs(err[i]))[:m]
        xs = np.sort(grid[idx])
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez_relative()
    print("coefficients c0..c3:", ", ".join(f"{v:.9e}" for v in c))
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
