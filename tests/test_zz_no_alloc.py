"""gdpa_fwd_no_alloc: the forward for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc when they run the operator (a host
framework that keeps all device memory in its own pool and gives plug-ins no
allocator, or a serving loop that cannot pay for cudaMalloc's implicit
synchronisation).  gdpa_fwd_no_alloc takes only inputs and outputs and keeps
its scratch in a static device array inside the library.  These tests call it
through the C ABI and compare it with gdpa_fwd, which takes a caller-allocated
workspace, on two calls in a row (the second reuses the shared scratch), and
with the fp64 oracle for every head dim.  The file is named to be collected
last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import recsys_context_personalised_b200 as pkg
from recsys_context_personalised_b200 import gdpa as G
import synthetic as syn

TOL = {torch.float32: 1e-3, torch.bfloat16: 2e-2}


def _entry():
    lib = pkg.load()
    fn = lib.gdpa_fwd_no_alloc
    vp = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(G.Problem), vp, vp, vp, vp, vp, vp, vp]
    fn.restype = ctypes.c_int
    return fn


def _status():
    """gdpa_fwd_no_alloc_status: the device status word of the last call."""
    lib = pkg.load()
    fn = lib.gdpa_fwd_no_alloc_status
    fn.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32)]
    fn.restype = ctypes.c_int
    out = ctypes.c_int32(-1)
    assert fn(torch.cuda.current_stream().cuda_stream, ctypes.byref(out)) == 0
    return out.value


def test_rejects_problems_beyond_the_static_scratch():
    # 16 heads * (2^24 / 128 + 1024) tiles need far more than 2 MiB of tile list;
    # the size check comes before any CUDA call
    p = G.problem(1024, 16, 64, 2048, 1 << 24, 1 << 15, "softmax", 0.125, torch.bfloat16)
    assert G.fwd_workspace_bytes(p) > (2 << 20)
    assert _entry()(ctypes.byref(p), 4096, 4096, 4096, 4096, 4096, 4096, None) == 5


def _rel(a, b):
    a, b = a.float().cpu().numpy(), b.float().cpu().numpy()
    den = np.abs(b).max()
    return float(np.abs(a - b).max() / den) if den > 0 else float(np.abs(a).max())


@pytest.mark.gpu
@pytest.mark.parametrize("dh", [32, 64, 128])
@pytest.mark.parametrize("phi,dtype", [("softmax", torch.bfloat16), ("silu", torch.bfloat16),
                                       ("silu", torch.float32)])
def test_no_alloc_matches_gdpa_fwd_on_two_calls(phi, dtype, dh):
    fn = _entry()
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    for call, (n, m, seed) in enumerate((([130, 0, 17, 256], 200, 1), ([513, 64, 3], 130, 2))):
        d = syn.random_problem(seed, len(n), 2, dh, m, n, dtype=dtype, std=0.6)
        s = 1.0 / dh ** 0.5 if phi == "softmax" else 0.5
        q, k, v = (d[x].to(dev) for x in ("q", "k", "v"))
        off = torch.tensor(d["offsets"], dtype=torch.int32, device=dev)
        p = pkg.problem_for(q, k, d["offsets"], phi, s)
        o_ref, lse_ref = pkg.fwd(p, q, off, k, v)
        o = torch.full_like(q, float("nan"))
        lse = torch.full((2, q.shape[0]), float("nan"), device=dev) if phi == "softmax" else None
        rc = fn(ctypes.byref(p), q.data_ptr(), off.data_ptr(), k.data_ptr(), v.data_ptr(),
                o.data_ptr(), lse.data_ptr() if lse is not None else None, stream.cuda_stream)
        assert rc == 0, f"call {call}: {G.STATUS.get(rc, rc)}"
        torch.cuda.synchronize()
        assert _status() == 0, f"call {call}"
        assert _rel(o, o_ref) <= TOL[dtype], f"call {call}"
        ro, rl = oracle.fwd(d["q"], d["k"], d["v"], d["offsets"], phi, s)
        den = np.abs(ro).max()
        err = float(np.abs(o.float().cpu().numpy() - ro).max() / den)
        assert err <= TOL[dtype], f"call {call} vs oracle: {err:.3e}"
        if lse is not None:
            assert float((lse - lse_ref).abs().max()) <= 1e-2, f"call {call}"
            assert float(np.abs(lse.cpu().numpy() - rl).max()) <= 1e-2, f"call {call}"


@pytest.mark.gpu
def test_no_alloc_reports_bad_device_offsets():
    """Decreasing device offsets: the call returns GDPA_OK (the check runs on
    the device), and gdpa_fwd_no_alloc_status reports GDPA_ERR_INVALID_ARG;
    the next call with good offsets clears it."""
    fn = _entry()
    dev = torch.device("cuda:0")
    d = syn.random_problem(3, 3, 2, 64, 64, [10, 20, 30], dtype=torch.bfloat16)
    q, k, v = (d[x].to(dev) for x in ("q", "k", "v"))
    p = pkg.problem_for(q, k, d["offsets"], "silu", 1.0)
    o = torch.empty_like(q)
    stream = torch.cuda.current_stream().cuda_stream
    for offs, want in (([0, 25, 20, 60], 1), (d["offsets"], 0)):
        off = torch.tensor(offs, dtype=torch.int32, device=dev)
        rc = fn(ctypes.byref(p), q.data_ptr(), off.data_ptr(), k.data_ptr(), v.data_ptr(),
                o.data_ptr(), None, stream)
        assert rc == 0
        assert _status() == want
