"""Pins of the fp64 sliding-window self-attention oracle (causal window of
width w on each sample's jagged tokens), CPU only: torch's
scaled_dot_product_attention with an explicit band mask and with is_causal
for a window wider than every sample, torch autograd, the GDPA oracle on one
query row at a time, w = 1 closed forms, central differences, and planted
slips that must each break a pin."""
import math
import os
import tempfile

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "window_oracle.c")


def _problem(seed, n=(9, 0, 14, 1), h=2, dh=8):
    rng = np.random.default_rng(seed)
    off = np.concatenate([[0], np.cumsum(n)]).astype(np.int64)
    T = int(off[-1])
    f = lambda: rng.standard_normal((T, h, dh)).astype(np.float32)   # noqa: E731
    return f(), f(), f(), f(), off


def _rel(a, b):
    den = max(np.abs(b).max(), 1e-300)
    return float(np.abs(np.asarray(a) - np.asarray(b)).max() / den)


def _torch_window(q, k, v, off, w, s, causal_only=False):
    qt, kt, vt = (torch.from_numpy(x).double().requires_grad_(True) for x in (q, k, v))
    outs = []
    for b in range(len(off) - 1):
        t0, t1 = off[b], off[b + 1]
        if t1 == t0:
            continue
        qb, kb, vb = (x[t0:t1].transpose(0, 1) for x in (qt, kt, vt))   # [h, n, dh]
        n = t1 - t0
        if causal_only:
            ob = F.scaled_dot_product_attention(qb, kb, vb, is_causal=True, scale=s)
        else:
            i = torch.arange(n)
            mask = (i[None, :] <= i[:, None]) & (i[None, :] > i[:, None] - w)
            ob = F.scaled_dot_product_attention(qb, kb, vb, attn_mask=mask, scale=s)
        outs.append((t0, t1, ob.transpose(0, 1)))
    return qt, kt, vt, outs


@pytest.mark.parametrize("w", [1, 3, 8, 64])
def test_matches_masked_sdpa_and_autograd(w):
    q, k, v, g, off = _problem(1)
    s = 0.35
    o, _ = oracle.win_fwd(q, k, v, off, w, s)
    qt, kt, vt, outs = _torch_window(q, k, v, off, w, s)
    ref = np.zeros_like(o)
    L = 0
    for t0, t1, ob in outs:
        ref[t0:t1] = ob.detach().numpy()
        L = L + (ob * torch.from_numpy(g[t0:t1]).double()).sum()
    assert _rel(o, ref) < 1e-12
    L.backward()
    dq, dk, dv = oracle.win_bwd(q, k, v, g, off, w, s)
    for got, t in ((dq, qt), (dk, kt), (dv, vt)):
        assert _rel(got, t.grad.numpy()) < 1e-12


def test_wide_window_is_causal_attention():
    q, k, v, g, off = _problem(2, n=(20, 7))
    o, _ = oracle.win_fwd(q, k, v, off, 10000, 0.25)
    _, _, _, outs = _torch_window(q, k, v, off, 10000, 0.25, causal_only=True)
    for t0, t1, ob in outs:
        assert _rel(o[t0:t1], ob.detach().numpy()) < 1e-12


def test_rows_match_the_gdpa_oracle():
    """Each query row is GDPA softmax over the keys of its window."""
    q, k, v, g, off = _problem(3, n=(12, 5), h=2, dh=8)
    w, s = 4, 0.5
    o, lse = oracle.win_fwd(q, k, v, off, w, s)
    for b in range(2):
        for t in range(off[b], off[b + 1]):
            lo = max(off[b], t - w + 1)
            kk = np.ascontiguousarray(k[lo:t + 1].transpose(1, 0, 2))[None]
            vv = np.ascontiguousarray(v[lo:t + 1].transpose(1, 0, 2))[None]
            og, lg = oracle.fwd(q[t:t + 1], kk, vv, [0, 1], "softmax", s)
            assert _rel(o[t], og[0]) < 1e-13
            assert np.abs(lse[:, t] - lg[:, 0]).max() < 1e-12


def test_window_of_one_closed_form():
    q, k, v, g, off = _problem(4)
    o, lse = oracle.win_fwd(q, k, v, off, 1, 0.7)
    np.testing.assert_allclose(o, v.astype(np.float64), atol=1e-15)
    qk = np.einsum("thd,thd->ht", q.astype(np.float64), k.astype(np.float64))
    np.testing.assert_allclose(lse, 0.7 * qk, atol=1e-12)


def test_backward_matches_central_differences():
    q, k, v, g, off = _problem(5, n=(4, 3), h=1, dh=3)
    w, s = 2, 0.6
    dq, dk, dv = oracle.win_bwd(q, k, v, g, off, w, s)
    gd = g.astype(np.float64)

    def loss(a, b_, c):
        o, _ = oracle.win_fwd(a.astype(np.float32), b_.astype(np.float32), c.astype(np.float32),
                              off, w, s)
        return float((o * gd).sum())

    x = [q.astype(np.float64), k.astype(np.float64), v.astype(np.float64)]
    eps = 2.0 ** -10
    for idx, grad in enumerate((dq, dk, dv)):
        fd = np.zeros_like(x[idx])
        for i in range(x[idx].size):
            xp, xm = [y.copy() for y in x], [y.copy() for y in x]
            xp[idx].reshape(-1)[i] += eps
            xm[idx].reshape(-1)[i] -= eps
            fd.reshape(-1)[i] = (loss(*xp) - loss(*xm)) / (2 * eps)
        assert _rel(grad, fd) < 2e-5, idx


MUTANTS = {
    "window_off_by_one": ("const int64_t lo = t - w + 1;", "const int64_t lo = t - w;"),
    "no_sample_start": ("return lo > t0 ? lo : t0;", "return lo > 0 ? lo : 0;"),
    "dk_no_scale": ("dk[at + d] += scale * dA * (double)qt[d];", "dk[at + d] += dA * (double)qt[d];"),
    "dv_uses_dA": ("dv[at + d] += P[i] * (double)gt[d];", "dv[at + d] += dA * (double)gt[d];"),
}
PINS = (lambda: test_matches_masked_sdpa_and_autograd(3), test_rows_match_the_gdpa_oracle,
        test_window_of_one_closed_form)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    with tempfile.TemporaryDirectory() as d:
        msrc = os.path.join(d, "mutant.c")
        open(msrc, "w").write(src.replace(old, new))
        lib = oracle.win_load(oracle.build(force=True, src=msrc, out=os.path.join(d, "libm.so")))
        saved = oracle._win_lib
        oracle._win_lib = lib
        failed = 0
        try:
            for pin in PINS:
                try:
                    pin()
                except AssertionError:
                    failed += 1
        finally:
            oracle._win_lib = saved
    assert failed, f"mutant {name} passed every pin"
