"""Sliding-window self-attention (gdpa_window_fwd: causal window of width w on
each sample's jagged tokens) against the fp64 oracle, through the C ABI: O
and LSE element by element on jagged batches with empty samples, ragged
128-row tiles, windows narrower and wider than a tile and than a sample, and
odd head counts.  Bound: max|gpu - ref| / max|ref| <= 2e-2 for bf16 inputs
with fp32 accumulation; LSE to 1e-2 absolute."""
import numpy as np
import pytest
import torch

import oracle
import recsys_context_personalised_b200 as pkg

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = 2e-2


def _case(seed, n, h, dh):
    g = torch.Generator().manual_seed(seed)
    T = int(sum(n))
    q, k, v = (torch.randn(T, h, dh, generator=g).bfloat16() for _ in range(3))
    return q, k, v, np.concatenate([[0], np.cumsum(n)]).astype(np.int64)


@pytest.mark.parametrize("dh", [32, 64])
@pytest.mark.parametrize("w", [1, 37, 128, 200, 5000])
@pytest.mark.parametrize("n,h", [([130, 0, 17, 300, 1], 2), ([513, 64], 3), ([256], 1)])
def test_window_matches_oracle(n, h, w, dh):
    q, k, v, off = _case(len(n) + w + dh + h, n, h, dh)
    scale = 1.0 / dh ** 0.5
    offd = torch.tensor(off, dtype=torch.int32, device=DEV)
    o, lse = pkg.gdpa.window_fwd(q.to(DEV), offd, k.to(DEV), v.to(DEV), w, scale, off)
    torch.cuda.synchronize()
    ro, rl = oracle.win_fwd(q, k, v, off, w, scale)
    err = np.abs(o.float().cpu().numpy() - ro).max() / np.abs(ro).max()
    assert err <= TOL, err
    assert np.abs(lse.cpu().numpy() - rl).max() <= 1e-2


def test_window_output_guard():
    q, k, v, off = _case(3, [200, 50], 2, 64)
    T = int(off[-1])
    offd = torch.tensor(off, dtype=torch.int32, device=DEV)
    big = torch.full((T + 128, 2, 64), 7.0, dtype=torch.bfloat16, device=DEV)
    o = big[64:64 + T]
    pkg.gdpa.window_fwd(q.to(DEV), offd, k.to(DEV), v.to(DEV), 100, 0.125, off, o=o)
    torch.cuda.synchronize()
    assert (big[:64] == 7.0).all() and (big[64 + T:] == 7.0).all()


def _rel(x, r, scale_ref):
    """max|x - r| over the larger of max|r| and max|scale_ref|: with w = 1
    each token attends to itself alone, so dQ and dK are exactly zero and are
    judged against the magnitude of dV, the gradient of the same dO."""
    den = max(np.abs(r).max(), np.abs(scale_ref).max(), 1e-30)
    return float(np.abs(x.float().cpu().numpy() - r).max() / den)


@pytest.mark.parametrize("dh", [32, 64])
@pytest.mark.parametrize("w", [1, 37, 128, 200, 5000])
@pytest.mark.parametrize("n,h", [([130, 0, 17, 300, 1], 2), ([513, 64], 3), ([256], 1)])
def test_window_backward_matches_oracle(n, h, w, dh):
    """gdpa_window_bwd on the GPU forward's O and LSE against the oracle's
    dQ, dK, dV (key blocks whose window reaches several query tiles, blocks
    that end inside the next sample, empty samples)."""
    q, k, v, off = _case(len(n) * 3 + w + dh + h, n, h, dh)
    T = int(off[-1])
    g = torch.randn(T, h, dh, generator=torch.Generator().manual_seed(w + dh)).bfloat16()
    scale = 1.0 / dh ** 0.5
    offd = torch.tensor(off, dtype=torch.int32, device=DEV)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o, lse = pkg.gdpa.window_fwd(qd, offd, kd, vd, w, scale, off)
    dq, dk, dv = pkg.gdpa.window_bwd(qd, offd, kd, vd, o, lse, g.to(DEV), w, scale, off)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.win_bwd(q, k, v, g, off, w, scale)
    assert _rel(dq, rq, rv) <= TOL and _rel(dk, rk, rv) <= TOL and _rel(dv, rv, rv) <= TOL


def test_window_backward_guard():
    """dQ, dK, dV inside sentinel-filled buffers: nothing outside the T rows
    is written."""
    q, k, v, off = _case(11, [200, 50, 300], 2, 64)
    T = int(off[-1])
    g = torch.randn(T, 2, 64, generator=torch.Generator().manual_seed(2)).bfloat16()
    offd = torch.tensor(off, dtype=torch.int32, device=DEV)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o, lse = pkg.gdpa.window_fwd(qd, offd, kd, vd, 100, 0.125, off)
    bufs = [torch.full((T + 256, 2, 64), 5.0, dtype=torch.bfloat16, device=DEV) for _ in range(3)]
    pkg.gdpa.window_bwd(qd, offd, kd, vd, o, lse, g.to(DEV), 100, 0.125, off,
                        dq=bufs[0][128:128 + T], dk=bufs[1][128:128 + T], dv=bufs[2][128:128 + T])
    torch.cuda.synchronize()
    for b in bufs:
        assert (b[:128] == 5.0).all() and (b[128 + T:] == 5.0).all()
    rq, rk, rv = oracle.win_bwd(q, k, v, g, off, 100, 0.125)
    T_ = slice(128, 128 + T)
    assert _rel(bufs[0][T_], rq, rv) <= TOL and _rel(bufs[1][T_], rk, rv) <= TOL
    assert _rel(bufs[2][T_], rv, rv) <= TOL


def test_window_power_law_batch():
    """The first 128 samples of the power-law workload's lengths (32..4096),
    h = 16, dh = 64, w = 256: forward and backward against the oracle."""
    import synthetic as syn
    n = syn.lengths(syn.WORKLOADS[5])[:128]
    h, dh, w = 16, 64, 256
    q, k, v, off = _case(21, n, h, dh)
    T = int(off[-1])
    g = torch.randn(T, h, dh, generator=torch.Generator().manual_seed(4)).bfloat16()
    offd = torch.tensor(off, dtype=torch.int32, device=DEV)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o, lse = pkg.gdpa.window_fwd(qd, offd, kd, vd, w, 0.125, off)
    dq, dk, dv = pkg.gdpa.window_bwd(qd, offd, kd, vd, o, lse, g.to(DEV), w, 0.125, off)
    torch.cuda.synchronize()
    ro, rl = oracle.win_fwd(q, k, v, off, w, 0.125)
    assert _rel(o, ro, ro) <= TOL
    assert np.abs(lse.cpu().numpy() - rl).max() <= 1e-2
    rq, rk, rv = oracle.win_bwd(q, k, v, g, off, w, 0.125)
    assert _rel(dq, rq, rv) <= TOL and _rel(dk, rk, rv) <= TOL and _rel(dv, rv, rv) <= TOL


def test_window_backward_of_an_empty_batch():
    off = np.zeros(3, dtype=np.int64)
    offd = torch.tensor(off, dtype=torch.int32, device=DEV)
    z = torch.empty(0, 2, 64, dtype=torch.bfloat16, device=DEV)
    o, lse = pkg.gdpa.window_fwd(z, offd, z, z, 8, 0.125, off)
    dq, dk, dv = pkg.gdpa.window_bwd(z, offd, z, z, o, lse, z, 8, 0.125, off)
    torch.cuda.synchronize()
    assert dq.numel() == dk.numel() == dv.numel() == 0
