"""Coefficients of the FMA-pipe exp2 used by the attention kernel's softmax.

Method (written here from the published techniques, not from any library's code):

* Cody and Waite's range reduction (W. J. Cody, W. Waite, "Software Manual for the
  Elementary Functions", 1980): 2^x = 2^n * 2^f with n = round(x) and f = x - n in
  [-1/2, 1/2]. In the kernel n is obtained by adding and subtracting 1.5 * 2^23 in fp32
  (round to nearest), and 2^n is applied by adding n to the exponent field.
* Remez's exchange algorithm (E. Ya. Remez, 1934) for the degree-3 polynomial p that
  minimises the maximum relative error |p(f) / 2^f - 1| on [-1/2, 1/2].

Running this file prints the coefficients (c0, c1, c2, c3) and the achieved maximum
relative error; ``attn_tc.cuh`` carries the printed values. The error bound is checked
by tests/test_exp2_poly.py.
"""

from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez(degree: int = DEGREE, iters: int = 30):
    n = degree + 2
    # initial reference: Chebyshev extrema on [LO, HI]
    k = np.arange(n)
    x = (LO + HI) / 2 + (HI - LO) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    coef = None
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  (relative error equioscillation)
        A = np.zeros((n, n))
        for i, xi in enumerate(x):
            A[i, :degree + 1] = xi ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(A, 2.0 ** x)
        coef = sol[:degree + 1]
        err = np.polyval(coef[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extrema of the error between sign changes
        sgn = np.sign(err)
        idx = np.concatenate([[0], np.nonzero(np.diff(sgn))[0] + 1, [len(grid)]])
        ext = [a + int(np.argmax(np.abs(err[a:b]))) for a, b in zip(idx[:-1], idx[1:]) if b > a]
        if len(ext) < n:
            break
        # keep the n consecutive extrema with the largest minimum magnitude
        best = max(range(len(ext) - n + 1), key=lambda s: np.min(np.abs(err[ext[s:s + n]])))
        x = grid[ext[best:best + n]]
    err = np.polyval(coef[::-1], grid) / 2.0 ** grid - 1.0
    return coef, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez()
    print("coefficients c0..c3:", ", ".join(f"{v:.9e}" for v in c))
    print(f"max relative error on [-1/2, 1/2]: {e:.3e}")
    print("as fp32:", ", ".join(f"{np.float32(v)!r}" for v in c))
