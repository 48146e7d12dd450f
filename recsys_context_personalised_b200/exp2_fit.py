"""Fit of the polynomial behind the kernels' FMA-pipe exp2 (exp2_fma2).

The softmax kernels evaluate part of their exponentials without the MUFU
unit: 2^x = 2^n * 2^f with n = floor(x) and f in [0, 1), and 2^f from a cubic
c0 + c1 f + c2 f^2 + c3 f^3.  The coefficients minimise the largest relative
error max |p(f) / 2^f - 1| over [0, 1]; they come from the Remez exchange
algorithm below (E. Remez, 1934: solve p(x_i) - 2^x_i = (-1)^i E 2^x_i on
deg + 2 reference points, move the references to the extrema of the error
curve, repeat until they settle).

``python exp2_fit.py`` prints the coefficients rounded to fp32 and the error
bound; csrc/gdpa_internal.cuh holds the same numbers.
"""
from __future__ import annotations

import numpy as np


def remez_exp2(deg: int = 3, iters: int = 40, grid: int = 200001):
    """Coefficients c0..c_deg (low order first) and the max relative error."""
    n = deg + 2
    xs = np.linspace(0.0, 1.0, grid)
    fx = np.exp2(xs)
    ref = 0.5 - 0.5 * np.cos(np.pi * np.arange(n) / (n - 1))   # Chebyshev points on [0, 1]
    c = None
    for _ in range(iters):
        A = np.zeros((n, n))
        A[:, :deg + 1] = ref[:, None] ** np.arange(deg + 1)[None, :]
        A[:, deg + 1] = -((-1.0) ** np.arange(n)) * np.exp2(ref)
        sol = np.linalg.solve(A, np.exp2(ref))
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], xs) / fx - 1.0
        # alternating extrema of the error curve: local extrema, then per sign
        # run the largest one, then trim to n points from the smaller end
        d = np.diff(err)
        ext = [0] + [i for i in range(1, grid - 1) if d[i - 1] * d[i] <= 0] + [grid - 1]
        runs = []
        for i in ext:
            if runs and np.sign(err[i]) == np.sign(err[runs[-1]]):
                if abs(err[i]) > abs(err[runs[-1]]):
                    runs[-1] = i
            else:
                runs.append(i)
        while len(runs) > n:
            runs = runs[1:] if abs(err[runs[0]]) < abs(err[runs[-1]]) else runs[:-1]
        ref = xs[runs]
    err = np.polyval(c[::-1], xs) / fx - 1.0
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    coef, bound = remez_exp2()
    print("c0..c3 (fp32):", [float(np.float32(v)) for v in coef])
    print("max relative error on [0, 1]:", bound)
