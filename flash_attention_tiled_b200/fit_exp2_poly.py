"""Fit of the cubic that ``exp2_poly_x2`` (csrc/frt_device.cuh) uses for 2^f
on [-1/2, 1/2]: a Remez exchange on the relative error p(f) / 2^f - 1.

    python -m flash_attention_tiled_b200.fit_exp2_poly

prints the coefficients c0..c3 (p(f) = c0 + c1 f + c2 f^2 + c3 f^3) and the
largest relative error.  The CUDA code carries them as fp32 literals.

Method: start from a Chebyshev-like reference of deg + 2 points; each step
solves p(x_i) - 2^(x_i) = (-1)^i E 2^(x_i) for the coefficients and the
levelled error E, then moves the reference to the alternating extrema of the
error on a fine grid, until the extrema level out.
"""
from __future__ import annotations

import numpy as np


def fit(deg: int = 3, lo: float = -0.5, hi: float = 0.5, iters: int = 40,
        grid_points: int = 200001):
    """Coefficients c[0..deg] of the minimax-relative-error polynomial for
    2^x on [lo, hi], and its largest relative error on the grid."""
    n = deg + 2
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, grid_points)
    c = np.zeros(deg + 1)
    r = np.zeros_like(grid)
    for _ in range(iters):
        a = np.zeros((n, n))
        for i in range(n):
            a[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            a[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(a, 2.0 ** x)
        c = sol[:deg + 1]
        r = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # local extrema of the error, the two ends included
        ext = [0] + [k for k in range(1, len(grid) - 1)
                     if (r[k] - r[k - 1]) * (r[k + 1] - r[k]) <= 0] + [len(grid) - 1]
        # keep the largest of each run of equal sign, then trim to n points
        pts: list[int] = []
        for k in ext:
            if pts and np.sign(r[k]) == np.sign(r[pts[-1]]):
                if abs(r[k]) > abs(r[pts[-1]]):
                    pts[-1] = k
            else:
                pts.append(k)
        while len(pts) > n:
            if abs(r[pts[0]]) < abs(r[pts[-1]]):
                pts.pop(0)
            else:
                pts.pop()
        x = grid[pts]
    return c, float(np.abs(r).max())


if __name__ == "__main__":
    coeffs, err = fit()
    print("c0..c3 =", ", ".join(f"{v:.9g}" for v in coeffs))
    print(f"max relative error on [-1/2, 1/2]: {err:.3g}")
