"""Fit the polynomial p(f) ~ 2^f on [0, 1) used for part of the softmax
exponentials in prefill_sm100.cu (run: python exp2_poly_fit.py).

Method: Cody-Waite style range reduction 2^x = 2^floor(x) * 2^f, f = x - floor(x)
in [0, 1) (W. J. Cody and W. Waite, Software Manual for the Elementary
Functions, 1980), and a degree-3 polynomial for 2^f fitted here by a Remez
exchange on the relative error, with p(0) = 1 pinned so that 2^n is exact at
integers.  Prints the coefficients (fp32) and the achieved max relative error.
"""

import numpy as np


def fit(deg=3, iters=30):
    # p(f) = 1 + f * (c1 + c2 f + c3 f^2);  minimise max |p(f) / 2^f - 1| on [0, 1]
    n = deg  # unknowns c1..c3 plus the levelled error E -> deg + 1 equations
    xs = 0.5 - 0.5 * np.cos(np.pi * np.arange(n + 1) / n)  # initial reference
    for _ in range(iters):
        A = np.zeros((n + 1, n + 1))
        rhs = np.zeros(n + 1)
        for r, x in enumerate(xs):
            t = 2.0 ** x
            for j in range(n):
                A[r, j] = x ** (j + 1) / t
            A[r, n] = (-1.0) ** r
            rhs[r] = 1.0 - 1.0 / t
        sol = np.linalg.solve(A, rhs)
        c = sol[:n]
        grid = np.linspace(0.0, 1.0, 200001)
        err = (1.0 + sum(c[j] * grid ** (j + 1) for j in range(n))) / 2.0 ** grid - 1.0
        # new reference: alternating extrema of the error
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        ext = sorted(idx, key=lambda i: -abs(err[i]))[: n + 1]
        xs = np.sort(grid[ext])
    return c, np.max(np.abs(err))


if __name__ == "__main__":
    c, e = fit()
    c32 = c.astype(np.float32)
    g = np.linspace(0, 1, 100001)
    p32 = (np.float32(1) + g.astype(np.float32) * (c32[0] + g.astype(np.float32) * (c32[1] + g.astype(np.float32) * c32[2])))
    e32 = np.max(np.abs(p32.astype(np.float64) / 2.0 ** g - 1.0))
    print("c1, c2, c3 =", ", ".join(f"{float(x):.9g}f" for x in c32))
    print(f"max relative error: {e:.3e} (fp64 coefficients), {e32:.3e} (fp32)")
