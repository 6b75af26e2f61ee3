"""Coefficients of the polynomial 2^f on f in [-1/2, 1/2] used by the attention
kernel's FMA-pipe exp2 (Cody & Waite range reduction: 2^x = 2^n * 2^f with n
the nearest integer to x; the remaining 2^f from a polynomial).

The polynomial minimises the maximum RELATIVE error (Remez exchange on the
weighted error 1 - p(f) / 2^f).  Run this file to print the coefficients and
the error bound that the kernel header quotes.
"""
import numpy as np


def remez_relative(degree: int, lo=-0.5, hi=0.5, iters=60):
    f = lambda x: np.exp2(x)
    n = degree + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    x = (lo + hi) / 2 + (hi - lo) / 2 * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # solve p(x_i) + (-1)^i E f(x_i) = f(x_i) for coefficients and E
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = (-1) ** i * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[:degree + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: alternating extrema of the error
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        ext = grid[idx]
        e = err[idx]
        # keep n points with alternating sign and largest magnitude
        sel = []
        for xi, ei in zip(ext, e):
            if sel and np.sign(ei) == np.sign(sel[-1][1]):
                if abs(ei) > abs(sel[-1][1]):
                    sel[-1] = (xi, ei)
            else:
                sel.append((xi, ei))
        while len(sel) > n:
            if abs(sel[0][1]) < abs(sel[-1][1]):
                sel.pop(0)
            else:
                sel.pop()
        if len(sel) < n:
            break
        x = np.array([s[0] for s in sel])
    err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    for deg in (3, 4):
        c, e = remez_relative(deg)
        c32 = c.astype(np.float32)
        g = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
        p = np.zeros_like(g)
        for ci in c32[::-1]:
            p = p * g + ci
        e32 = float(np.abs(p.astype(np.float64) / np.exp2(g.astype(np.float64)) - 1).max())
        print(f"degree {deg}: max rel err {e:.3e} (fp32 Horner {e32:.3e})")
        print("  c0..c%d = %s" % (deg, ", ".join(f"{float(v):.9e}f" for v in c32)))
