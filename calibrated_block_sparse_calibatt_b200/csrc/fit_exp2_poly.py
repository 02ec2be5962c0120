"""Derives the coefficients of the FMA-pipe exp2 used by the tensor-core softmax.

Method (Cody and Waite's argument reduction, then a polynomial on the reduced
argument): 2^x = 2^n * 2^f with n an integer near x and f = x - n small.  2^f is
approximated by a polynomial chosen to minimise the maximum relative error on
the reduced interval (Remez exchange, equioscillation of the relative error on
degree + 2 points), here computed with numpy from scratch: a cubic for the
attention softmax and a quintic for the offline energy passes.  The
kernel rounds to nearest (n = rint(x), f in [-1/2, 1/2]) using the float
addition of 1.5 * 2^23, so no float-to-integer conversion instruction is used.  The
cubic only feeds bf16 attention probabilities (8-bit mantissa), so a relative
error near 1e-4 is far below their rounding step; the quintic's 7.5e-8 is under
one float32 ulp (1.2e-7 relative), for the energies' float32 sums.

Run: python fit_exp2_poly.py  -> prints the coefficients and the error bound.
"""

import numpy as np


def remez_relative(degree=3, iters=60, lo=-0.5, hi=0.5):
    # initial reference: Chebyshev extrema mapped to [lo, hi]
    m = degree + 2
    xs = lo + (hi - lo) * (0.5 - 0.5 * np.cos(np.pi * np.arange(m) / (m - 1)))
    grid = np.linspace(lo, hi, 400001)
    for _ in range(iters):
        # solve sum c_k x^k - 2^x = (-1)^i E 2^x  (relative error equioscillates)
        a = np.zeros((m, m))
        for i, x in enumerate(xs):
            a[i, :degree + 1] = x ** np.arange(degree + 1)
            a[i, degree + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(a, 2.0 ** xs)
        c = sol[:degree + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: one extremum per interval of constant error sign, then
        # the m consecutive (alternating) ones whose smallest magnitude is largest
        sign = np.sign(err)
        segments = np.split(np.arange(len(grid)), np.nonzero(sign[1:] != sign[:-1])[0] + 1)
        ext = [seg[np.argmax(np.abs(err[seg]))] for seg in segments]
        if len(ext) < m:
            break
        first = max(range(len(ext) - m + 1), key=lambda i: np.abs(err[ext[i:i + m]]).min())
        xs = grid[ext[first:first + m]]
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    for degree, use in ((3, "attention probabilities (bf16)"), (5, "offline energy sums (float32)")):
        c, e = remez_relative(degree)
        print(f"degree {degree}, {use}: c0..c{degree} =", ", ".join(f"{v:.9e}" for v in c))
        print(f"  max relative error on [-1/2, 1/2]: {e:.3e}")
