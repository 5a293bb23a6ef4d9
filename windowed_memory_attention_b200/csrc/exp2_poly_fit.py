"""Coefficients of the FMA-pipe 2^x used by the attention kernel.

Method: range reduction x = j + f with j = round-to-nearest(x) and
f in [-1/2, 1/2] (Cody and Waite, "Software Manual for the Elementary
Functions", 1980, additive argument reduction), then a degree-3 polynomial
p(f) ~ 2^f that minimises the maximum relative error on [-1/2, 1/2], found with
the Remez exchange algorithm (Remez 1934).  The kernel forms 2^j by adding j to
the exponent field of p(f).

Run ``python exp2_poly_fit.py`` to print the coefficients and the error bound;
``tests/test_exp2_poly.py`` checks the constants in ``attend_sm100.cu`` against
this fit and the bound against float32 evaluation.
"""
import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez(degree=DEGREE, iters=30):
    n = degree + 2
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^{x_i} = (-1)^i E 2^{x_i} for the coefficients and E
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:degree + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: one extremum of the error per sign-alternating segment
        sgn = np.sign(err)
        idx = [0]
        for i in range(1, len(grid)):
            if sgn[i] != sgn[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        idx = np.array(idx)
        if len(idx) < n:
            break
        # keep the n consecutive extrema with the largest minimum magnitude
        best = max(range(len(idx) - n + 1), key=lambda s: np.abs(err[idx[s:s + n]]).min())
        x = grid[idx[best:best + n]]
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez()
    for i, v in enumerate(c):
        print(f"c{i} = {np.float32(v).item()!r:>14}  ({float(np.float32(v)).hex()})")
    print(f"max relative error on [{LO}, {HI}]: {e:.3e}")
