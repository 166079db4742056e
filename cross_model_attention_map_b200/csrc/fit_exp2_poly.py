"""Coefficients of the FMA-pipe 2^x in exp2_fma.cuh.

2^f on [-1/2, 1/2] by the polynomial of degree 5 that minimises the maximum relative error
max |p(f) / 2^f - 1| (Remez exchange algorithm: solve for the polynomial that equioscillates on a
reference of deg + 2 points, move the reference to the extrema of the new error curve, repeat).
The result is printed as C float literals for the header; the error bound it reaches (7.5e-8
before fp32 rounding of the coefficients and of the evaluation) is what tests/test_exp2_poly.py
checks the header's coefficients against.

usage: python fit_exp2_poly.py [degree]
"""
import sys

import numpy as np


def remez_exp2(deg: int, lo: float = -0.5, hi: float = 0.5, iters: int = 40):
    """Minimax coefficients c[0..deg] (ascending powers) of 2^f on [lo, hi], relative error."""
    n = deg + 2
    ref = (lo + hi) / 2 - (hi - lo) / 2 * np.cos(np.pi * np.arange(n) / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    c = None
    for _ in range(iters):
        a = np.zeros((n, n))
        for i, x in enumerate(ref):
            a[i, :deg + 1] = x ** np.arange(deg + 1)
            a[i, deg + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(a, 2.0 ** ref)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # local extrema of the error curve (and both ends), then one point per sign run
        d = np.diff(err)
        turn = np.where(d[:-1] * d[1:] <= 0)[0] + 1
        idx = np.concatenate(([0], turn, [len(grid) - 1]))
        runs = []
        for j in idx:
            if runs and np.sign(err[j]) == np.sign(err[runs[-1]]):
                if abs(err[j]) > abs(err[runs[-1]]):
                    runs[-1] = j
            else:
                runs.append(j)
        while len(runs) > n:
            runs.pop(0 if abs(err[runs[0]]) < abs(err[runs[-1]]) else -1)
        if len(runs) != n:
            break
        ref = grid[runs]
    err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 5
    coef, e = remez_exp2(deg)
    print("// max relative error %.3e (exact arithmetic)" % e)
    for k, ck in enumerate(coef):
        print("constexpr float kExp2C%d = %.9ef;" % (k, np.float32(ck)))
