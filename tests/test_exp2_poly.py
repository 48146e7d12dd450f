"""The FMA-pipe exp2 of the softmax kernels (Cody-Waite reduction and a cubic
minimax polynomial): its coefficients come from the committed Remez fit, the
method's error bound holds (CPU), and the device function meets it against
numpy's exp2 over a dense sweep (GPU, through the C ABI)."""
import ctypes
import os
import re

import numpy as np
import pytest

from recsys_context_personalised_b200 import exp2_fit

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "recsys_context_personalised_b200", "csrc", "gdpa_internal.cuh")
BOUND = 7.5e-5


def _kernel_coefficients():
    src = open(HDR).read()
    return [float(re.search(rf"kExp2C{i} = ([0-9.]+)f", src).group(1)) for i in range(4)]


def test_remez_fit_reproduces_the_kernel_coefficients():
    coef, bound = exp2_fit.remez_exp2()
    assert bound <= BOUND
    assert np.allclose(_kernel_coefficients(), coef, rtol=0, atol=5e-8)


def test_remez_error_equioscillates():
    """A minimax fit of degree 3 touches its error bound at 5 alternating points."""
    coef, bound = exp2_fit.remez_exp2()
    xs = np.linspace(0, 1, 200001)
    err = np.polyval(coef[::-1], xs) / np.exp2(xs) - 1
    assert abs(err[0]) == pytest.approx(bound, rel=1e-3)
    assert abs(err[-1]) == pytest.approx(bound, rel=1e-3)
    peaks = [i for i in range(1, len(xs) - 1) if abs(err[i]) >= abs(err[i - 1]) and
             abs(err[i]) >= abs(err[i + 1]) and abs(err[i]) > 0.99 * bound]
    assert len(peaks) == 3


def _emulate(x):
    """The kernel's steps in float32 (numpy), to pin the range reduction."""
    c0, c1, c2, c3 = (np.float32(v) for v in _kernel_coefficients())
    x = np.maximum(x.astype(np.float32), np.float32(-126))
    n = np.floor(x)
    f = (x - n).astype(np.float32)
    q = ((c3 * f + c2) * f + c1) * f + c0
    bits = q.view(np.uint32).astype(np.int64) + (n.astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_range_reduction_meets_the_bound_on_the_softmax_range():
    x = np.linspace(-125, 8, 2_000_001, dtype=np.float32)
    y = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y / ref - 1)) <= 1.2 * BOUND      # + fp32 rounding of the Horner steps
    # below -125 the result has the subnormal exponent and loses low mantissa bits
    x = np.linspace(-126, -125, 10001, dtype=np.float32)
    assert np.max(np.abs(_emulate(x) / np.exp2(x.astype(np.float64)) - 1)) <= 1e-3
    tiny = _emulate(np.array([-126.5, -200.0, -1e30, -np.inf], dtype=np.float32))
    assert np.all(tiny >= 0) and np.all(tiny <= 2.0 ** -125)


@pytest.mark.gpu
def test_device_exp2_against_numpy():
    import torch
    import recsys_context_personalised_b200 as pkg
    lib = pkg.load()
    fn = lib.gdpa_selftest_exp2
    fn.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    x = torch.linspace(-125, 8, 4_000_001, dtype=torch.float32, device="cuda:0")
    y_fma, y_mufu = torch.empty_like(x), torch.empty_like(x)
    assert fn(x.data_ptr(), y_fma.data_ptr(), y_mufu.data_ptr(), x.numel(),
              torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    ref = np.exp2(x.cpu().double().numpy())
    rel_fma = np.abs(y_fma.cpu().double().numpy() / ref - 1)
    rel_mufu = np.abs(y_mufu.cpu().double().numpy() / ref - 1)
    assert rel_fma.max() <= 1.2 * BOUND, rel_fma.max()
    # the polynomial is well below bf16's half-ulp (2^-9), like the hardware unit
    assert rel_mufu.max() <= 2.0 ** -20
    # the device fuses the Horner steps (one rounding per step instead of two),
    # so it matches the float32 emulation to a few ulps, not bit for bit
    emu = _emulate(x.cpu().numpy()).astype(np.float64)
    assert np.max(np.abs(y_fma.cpu().double().numpy() / emu - 1)) <= 2.0 ** -21
