"""Fit of the polynomial behind the kernels' GELU (gelu_f, gelu_grad).

GELU(x) = x * Phi(x) with Phi(x) = (1 + erf(x / sqrt 2)) / 2, so

    GELU(x) = x / 2 + |x| * t * h(t^2),   t = min(|x| / sqrt 2, Z),   h(u) = erf(sqrt u) / (2 sqrt u),

because erf is odd and x * erf(x / sqrt 2) = |x| * erf(|x| / sqrt 2).  h is smooth on
[0, Z^2]; it is evaluated in the centred variable s = 2 t^2 / Z^2 - 1 in [-1, 1] as a
polynomial of degree 12 whose monomial coefficients stay below 0.2, so that Horner's
rule in fp32 loses nothing against the fit.  The polynomial interpolates h at the
Chebyshev-Lobatto points of [-1, 1] (the extrema of T_12; interpolation there is
within a small factor of the minimax polynomial), except that at s = 1 it takes the
value 1 / (2 Z), so that erf(Z) reads exactly 1: past |x| = Z sqrt 2 (erf(3.6) =
1 - 3.6e-7), GELU(x) is x or 0 to within fp32 rounding.

``python gelu_fit.py`` prints the coefficients rounded to fp32 and the largest error of
the fp32 evaluation against the exact GELU; csrc/gdpa_internal.cuh holds the same numbers.
"""
from __future__ import annotations

import math

import numpy as np

Z = 3.6
DEG = 12


def _h(s: np.ndarray) -> np.ndarray:
    """h at u = Z^2 (s + 1) / 2: erf(sqrt u) / (2 sqrt u), 1 / sqrt(pi) at u = 0."""
    t = Z * np.sqrt((s + 1.0) / 2.0)
    out = np.empty_like(t)
    small = t < 1e-8
    out[small] = 1.0 / math.sqrt(math.pi)
    tt = t[~small]
    out[~small] = np.array([math.erf(v) for v in tt]) / (2.0 * tt)
    return out


def fit(deg: int = DEG) -> np.ndarray:
    """Monomial coefficients c0..c_deg (low order first) in s."""
    s = np.cos(np.pi * np.arange(deg + 1) / deg)       # Chebyshev-Lobatto points, s[0] = 1
    y = _h(s)
    y[0] = 1.0 / (2.0 * Z)                            # erf(Z) := 1
    return np.polynomial.polynomial.polyfit(s, y, deg)


def gelu_fp32(x: np.ndarray, c32: np.ndarray) -> np.ndarray:
    """The kernels' evaluation order in fp32 (numpy emulation)."""
    x = np.asarray(x, dtype=np.float32)
    ax = np.abs(x)
    t = np.minimum(ax * np.float32(1.0 / math.sqrt(2.0)), np.float32(Z))
    s = (t * t * np.float32(2.0 / (Z * Z)) - np.float32(1.0)).astype(np.float32)
    p = np.full_like(s, c32[-1])
    for cc in c32[-2::-1]:
        p = (p * s + cc).astype(np.float32)
    return (np.float32(0.5) * x + ax * t * p).astype(np.float32)


def gelu_exact(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    return np.array([0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))) for v in x.ravel()]).reshape(
        x.shape)


if __name__ == "__main__":
    c = fit()
    c32 = c.astype(np.float32)
    print("c0..c12 (fp32):", [float(v) for v in c32])
    xs = np.linspace(-10.0, 10.0, 200001)
    err = np.abs(gelu_fp32(xs, c32).astype(np.float64) - gelu_exact(xs)).max()
    print("max |GELU_fp32 - GELU| on [-10, 10]:", err)
