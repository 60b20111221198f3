"""Coefficients of the polynomial exp2 used by the attention kernels (ptx.cuh, exp2_poly2).

    python -m latent_kv_attention_down_b200.exp2_fit

The kernels split 2^y into 2^round(y) (exponent field) and 2^f, f in [-1/2, 1/2].
This script finds the degree-3 polynomial p minimising max |p(f) - 2^f| / 2^f on
that interval by the Remez exchange algorithm (equioscillation of the relative
error at d + 2 points), rounds the coefficients to fp32 and reports the maximum
relative error of the rounded polynomial on a fine grid.
"""
from __future__ import annotations

import numpy as np


def remez_exp2(degree: int = 3, lo: float = -0.5, hi: float = 0.5, iters: int = 30):
    n = degree + 2
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        a = np.zeros((n, n))
        for i in range(n):
            a[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            a[i, degree + 1] = -((-1) ** i) * np.exp2(x[i])
        coef = np.linalg.solve(a, np.exp2(x))[:degree + 1]
        err = (np.polyval(coef[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        sign = np.sign(err)
        ext = [0]
        for k in range(1, len(grid)):
            if sign[k] != sign[ext[-1]]:
                ext.append(k)
            elif abs(err[k]) > abs(err[ext[-1]]):
                ext[-1] = k
        while len(ext) > n:
            ext.pop(0 if abs(err[ext[0]]) < abs(err[ext[-1]]) else -1)
        if len(ext) == n:
            x = grid[ext]
    return coef


def main():
    coef = remez_exp2().astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 100001)
    rel = np.abs(np.polyval(coef[::-1].astype(np.float64), grid) - np.exp2(grid)) / np.exp2(grid)
    for i, c in enumerate(coef):
        print(f"c{i} = {float(c)!r}")
    print(f"max relative error (fp32 coefficients): {rel.max():.3e}")


if __name__ == "__main__":
    main()
