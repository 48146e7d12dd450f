"""The kernels' GELU polynomial (gdpa_internal.cuh kGeluH, fitted by
recsys_context_personalised_b200/gelu_fit.py): its coefficients are the fit's,
and its fp32 evaluation, emulated step by step in numpy, stays within 4e-6 of
the exact x * Phi(x) computed with the C library's erf."""
import math
import os
import re

import numpy as np

from recsys_context_personalised_b200 import gelu_fit

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_coefficients():
    src = open(os.path.join(ROOT, "recsys_context_personalised_b200", "csrc",
                            "gdpa_internal.cuh")).read()
    body = re.search(r"kGeluH\[13\]\s*=\s*\{([^}]*)\}", src).group(1)
    return np.array([float(v.strip().rstrip("f")) for v in body.split(",")], dtype=np.float32)


def test_header_holds_the_fitted_coefficients():
    assert np.array_equal(_header_coefficients(), gelu_fit.fit().astype(np.float32))


def test_fp32_polynomial_gelu_is_within_4e6_of_the_exact_gelu():
    c32 = _header_coefficients()
    xs = np.concatenate([np.linspace(-10.0, 10.0, 100001), [0.0, 1e-30, -1e-30, 5.09, -5.09]])
    got = gelu_fit.gelu_fp32(xs, c32).astype(np.float64)
    exact = np.array([0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0))) for v in xs])
    assert np.abs(got - exact).max() <= 4e-6


def test_tails_are_x_and_zero():
    """Past |x| = Z sqrt 2 the fit reads erf = 1: GELU(x) = x for large x and 0
    for very negative x, to within fp32 rounding of the product."""
    c32 = _header_coefficients()
    for x in (6.0, 50.0, 1e4):
        assert abs(gelu_fit.gelu_fp32(np.array([x]), c32)[0] - x) <= 1e-6 * x
        assert abs(gelu_fit.gelu_fp32(np.array([-x]), c32)[0]) <= 1e-6 * x


def test_gelu_derivative_pieces_are_consistent():
    """The backward's Phi(x) = 1/2 + sign(x) t h(t^2) matches (1 + erf(x/sqrt 2))/2."""
    c32 = _header_coefficients()
    xs = np.linspace(-9.0, 9.0, 20001).astype(np.float32)
    ax = np.abs(xs)
    t = np.minimum(ax * np.float32(1 / math.sqrt(2)), np.float32(gelu_fit.Z))
    s = t * t * np.float32(2 / gelu_fit.Z ** 2) - np.float32(1)
    p = np.full_like(s, c32[-1])
    for cc in c32[-2::-1]:
        p = p * s + cc
    cdf = 0.5 + np.copysign(t * p, xs)
    exact = np.array([0.5 * (1 + math.erf(v / math.sqrt(2))) for v in xs.astype(np.float64)])
    assert np.abs(cdf - exact).max() <= 2e-6
