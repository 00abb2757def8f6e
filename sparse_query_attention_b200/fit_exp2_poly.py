"""Derives the degree-3 polynomial for 2^f, f in [-1/2, 1/2], that the
kernels use to take part of the softmax exponentials off the MUFU.

Method: Remez exchange for the minimax approximation under relative error
(linear system on n+2 alternating points, then the extrema of the error
become the next points).  Prints the coefficients c0..c3 and the maximum
relative error; the kernels carry the printed values as kExp2C0..kExp2C3.

    python -m sparse_query_attention_b200.fit_exp2_poly
"""

from __future__ import annotations

import numpy as np


def remez_exp2(deg: int = 3, lo: float = -0.5, hi: float = 0.5, iters: int = 30):
    n = deg + 2
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    coef, err_max = None, None
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(deg + 1):
            A[:, i] = x ** i
        A[:, deg + 1] = (-1.0) ** np.arange(n) * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(x))
        coef = sol[:deg + 1]
        err = (np.polyval(coef[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        err_max = float(np.abs(err).max())
        cand = [0] + [i for i in range(1, len(grid) - 1)
                      if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0] + [len(grid) - 1]
        sel = []
        for i in cand:
            if not sel or np.sign(err[i]) != np.sign(err[sel[-1]]):
                sel.append(i)
            elif abs(err[i]) > abs(err[sel[-1]]):
                sel[-1] = i
        while len(sel) > n:
            sel.pop(0 if abs(err[sel[0]]) < abs(err[sel[-1]]) else -1)
        if len(sel) < n:
            break
        x = grid[sel]
    return [float(c) for c in coef], err_max


if __name__ == "__main__":
    c, e = remez_exp2()
    print("coefficients:", c)
    print("max relative error:", e)
