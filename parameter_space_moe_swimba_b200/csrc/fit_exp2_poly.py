"""Fit the polynomial p(f) ~ 2^f on [-1/2, 1/2] used by the scan kernel's FMA-pipe exp2.

2^x = 2^j * 2^f with j = round(x), f = x - j in [-1/2, 1/2]. The coefficients are a minimax fit of
the RELATIVE error (Remez exchange on the Chebyshev nodes, float64), then rounded to float32. The
script prints the coefficients and the max relative error of the float32 Horner evaluation on a
dense grid, which the CUDA code's comment quotes.

    python parameter_space_moe_swimba_b200/csrc/fit_exp2_poly.py [degree]
"""
import sys

import numpy as np


def remez_relative(deg, iters=30):
    a, b = -0.5, 0.5
    n = deg + 2
    # initial reference: Chebyshev extrema
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    f = lambda t: np.exp2(t)
    for _ in range(iters):
        # solve p(x_i) - f(x_i) = (-1)^i E f(x_i)  (relative equioscillation)
        V = np.vander(x, deg + 1, increasing=True)
        M = np.hstack([V, -((-1.0) ** np.arange(n))[:, None] * f(x)[:, None]])
        sol = np.linalg.solve(M, f(x))
        c = sol[:-1]
        grid = np.linspace(a, b, 200001)
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        # new reference: extrema of the error between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        cand = grid[idx]
        ecand = err[idx]
        # keep n alternating points with the largest errors
        order = np.argsort(cand)
        cand, ecand = cand[order], ecand[order]
        pts = [0]
        for i in range(1, len(cand)):
            if np.sign(ecand[i]) == np.sign(ecand[pts[-1]]):
                if abs(ecand[i]) > abs(ecand[pts[-1]]):
                    pts[-1] = i
            else:
                pts.append(i)
        while len(pts) > n:
            # drop the smaller end
            if abs(ecand[pts[0]]) < abs(ecand[pts[-1]]):
                pts.pop(0)
            else:
                pts.pop()
        if len(pts) < n:
            break
        x = cand[pts]
    return c


def f32_horner_error(c32):
    grid = np.linspace(-0.5, 0.5, 2_000_001).astype(np.float32)
    p = np.full_like(grid, c32[-1])
    for ck in c32[-2::-1]:
        p = (p * grid + ck).astype(np.float32)  # numpy float32 ops round each step
    ref = np.exp2(grid.astype(np.float64))
    return float(np.max(np.abs(p.astype(np.float64) - ref) / ref))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 5
    c = remez_relative(deg)
    c32 = c.astype(np.float32)
    for i, ci in enumerate(c32):
        print(f"c{i} = {float(ci).hex()}  ({ci:.9e})")
    print(f"max relative error of the float32 Horner evaluation on [-1/2, 1/2]: {f32_horner_error(c32):.3e}")
