"""Fit the cubic used by exp2_poly.cuh: p(f) ~ 2^f on [-1/2, 1/2], minimising
the maximum RELATIVE error by the Remez exchange algorithm (equioscillation
of the weighted error at degree + 2 points), then rounding the coefficients
to float32.

    python fit_exp2_poly.py      # prints the coefficients and the error bound
"""
import numpy as np

DEG = 3
A, B = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    # start from Chebyshev extrema
    x = 0.5 * (A + B) + 0.5 * (B - A) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(A, B, 200001)
    for _ in range(iters):
        f = np.exp2(x)
        # solve sum_k c_k x^k + (-1)^i E f(x_i) = f(x_i)   (relative weight 1/f)
        M = np.zeros((n, n))
        for k in range(deg + 1):
            M[:, k] = x ** k
        M[:, deg + 1] = (-1.0) ** np.arange(n) * f
        sol = np.linalg.solve(M, f)
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # new reference: extrema of err between sign changes
        idx = []
        sgn = np.sign(err)
        start = 0
        for i in range(1, len(grid) + 1):
            if i == len(grid) or sgn[i] != sgn[start]:
                seg = np.arange(start, i)
                idx.append(seg[np.argmax(np.abs(err[seg]))])
                start = i
        if len(idx) >= n:
            idx = sorted(idx, key=lambda j: -abs(err[j]))[:n]
            x = np.sort(grid[idx])
    return c, np.abs(err).max()


if __name__ == "__main__":
    c, e = remez()
    c32 = c.astype(np.float32)
    g = np.linspace(A, B, 200001).astype(np.float32)
    p = np.float32(c32[3])
    for k in (2, 1, 0):
        p = (p * g + c32[k]).astype(np.float32)
    rel = np.abs(p.astype(np.float64) - np.exp2(g.astype(np.float64))) / np.exp2(g.astype(np.float64))
    for k, v in enumerate(c32):
        print(f"c{k} = {float(v):.9e}f  ({float(v).hex()})")
    print(f"max relative error: minimax {e:.3e}, float32 evaluation {rel.max():.3e}")
