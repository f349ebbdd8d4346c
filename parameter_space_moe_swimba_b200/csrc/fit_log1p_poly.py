"""Fit the polynomial q(e) ~ log1p(e) / e on [0, 1] used by the projection epilogue's softplus.

softplus(v) = max(v, 0) + log1p(e) with e = exp(-|v|) in (0, 1]; log1p(e) = e * q(e) keeps full
relative accuracy for small e (where 1 + e would round away e's low bits) without a branch and
without a second special-function instruction. The coefficients are a minimax fit of the RELATIVE
error (Remez exchange, float64), then rounded to float32; the script prints them and the max
relative error of log1p(e) = e * q(e) evaluated by float32 Horner on a dense grid.

    python parameter_space_moe_swimba_b200/csrc/fit_log1p_poly.py [degree]
"""
import sys

import numpy as np


def target(e):
    return np.where(e == 0.0, 1.0, np.log1p(e) / np.where(e == 0.0, 1.0, e))


def remez_relative(deg, a=0.0, b=1.0, iters=40):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, 200001)
    c = None
    for _ in range(iters):
        V = np.vander(x, deg + 1, increasing=True)
        fx = target(x)
        M = np.hstack([V, -((-1.0) ** np.arange(n))[:, None] * fx[:, None]])
        sol = np.linalg.solve(M, fx)
        c = sol[:-1]
        err = (np.polyval(c[::-1], grid) - target(grid)) / target(grid)
        idx = [0] + [i for i in range(1, len(grid) - 1) if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0]
        idx.append(len(grid) - 1)
        cand, ecand = grid[idx], err[idx]
        pts = [0]
        for i in range(1, len(cand)):
            if np.sign(ecand[i]) == np.sign(ecand[pts[-1]]):
                if abs(ecand[i]) > abs(ecand[pts[-1]]):
                    pts[-1] = i
            else:
                pts.append(i)
        while len(pts) > n:
            if abs(ecand[pts[0]]) < abs(ecand[pts[-1]]):
                pts.pop(0)
            else:
                pts.pop()
        if len(pts) < n:
            break
        x = cand[pts]
    return c


def f32_error(c32):
    e = np.concatenate([np.linspace(0.0, 1.0, 2_000_001), np.logspace(-30, 0, 200001)]).astype(np.float32)
    q = np.float32(c32[-1])
    for cc in c32[-2::-1]:
        q = (q * e + np.float32(cc)).astype(np.float32)
    got = (e * q).astype(np.float64)
    ref = np.log1p(e.astype(np.float64))
    m = ref > 0
    return float(np.max(np.abs(got[m] - ref[m]) / ref[m]))


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 7
    c = remez_relative(deg)
    c32 = [np.float32(v) for v in c]
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v).hex()}  ({float(v):.9g})")
    print(f"float32 Horner max relative error of log1p: {f32_error(c32):.3g}")


if __name__ == "__main__":
    main()
