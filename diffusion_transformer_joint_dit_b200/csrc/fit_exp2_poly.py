"""Fit the polynomial the attention softmax uses for part of its exp2 calls.

exp2(x) = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]
(Cody-Waite style range reduction; n is added to the exponent field).  2^f
is approximated by a degree-3 polynomial p(f) chosen to minimise the
maximum *relative* error on [-1/2, 1/2] with the Remez exchange algorithm,
started from Chebyshev nodes.  The softmax stores P in bf16 (8 significant
bits) or fp16 (11 bits), so a relative error near 2^-13 is ample.

Run:  python fit_exp2_poly.py   (prints the coefficients and the error)
The printed float32 coefficients are kPolyC0..kPolyC3 in softmax_sm100.cuh.
"""

import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez_relative(deg, lo, hi, iters=30):
    n = deg + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    f = lambda t: np.exp2(t)
    c = None
    for _ in range(iters):
        # Solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative equioscillation)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        sign = np.sign(err)
        idx = np.concatenate(([0], np.nonzero(np.diff(sign))[0] + 1, [len(grid)]))
        new = []
        for a, b in zip(idx[:-1], idx[1:]):
            j = a + np.argmax(np.abs(err[a:b]))
            new.append(grid[j])
        if len(new) != n:
            break
        x = np.array(new)
    return c, np.max(np.abs(err))


if __name__ == "__main__":
    c, e = remez_relative(DEG, LO, HI)
    c32 = c.astype(np.float32)
    grid = np.linspace(LO, HI, 100001)
    p32 = np.zeros_like(grid, dtype=np.float32)
    for coef in c32[::-1]:
        p32 = p32 * grid.astype(np.float32) + coef
    e32 = np.max(np.abs(p32.astype(np.float64) / np.exp2(grid) - 1))
    print("coefficients c0..c3 (float32):", ", ".join(f"{v:.9e}f" for v in c32))
    print(f"max relative error: {e:.3e} (float64 coefficients), {e32:.3e} (float32 Horner)")
