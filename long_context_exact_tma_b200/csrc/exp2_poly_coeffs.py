"""Derives the coefficients of the software exp2 in usp_ptx.cuh (exp2_poly2).

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2]
(Cody and Waite's argument reduction); 2^f is a degree-3 polynomial whose
maximum RELATIVE error on [-1/2, 1/2] is minimal, found with the Remez exchange
algorithm below. Run it to print the coefficients (fp32) and the error bound;
the kernels carry the printed values.
"""
import numpy as np


def remez_exp2(degree=3, a=-0.5, b=0.5, iters=60):
    m = degree + 2
    x = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * np.arange(m)[::-1] / (m - 1))
    grid = np.linspace(a, b, 400001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i at the m reference points
        A = np.zeros((m, m))
        for i in range(m):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = (-1) ** i * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:degree + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1
        segs = np.split(np.arange(len(grid)), np.where(np.diff(np.sign(err)) != 0)[0] + 1)
        pts = [seg[np.argmax(np.abs(err[seg]))] for seg in segs]
        if len(pts) != m:
            break
        x = grid[pts]
    c32 = c.astype(np.float32)
    err32 = np.abs(np.polyval(c32[::-1].astype(np.float64), grid) / 2.0 ** grid - 1).max()
    return c32, err32


if __name__ == "__main__":
    c, e = remez_exp2()
    print("coefficients c0..c3:", ", ".join(f"{float(v):.9g}f" for v in c))
    print(f"max relative error on [-1/2, 1/2]: {e:.3g}")
