"""Pins of the fp64 seed-query attention pooling oracle (first level of HSP:
learned seeds attend over each sample's tokens), CPU only: the GDPA oracle
with the roles swapped (seeds as the queries of a one-sample problem, the
sample's tokens as its keys and values), torch's scaled_dot_product_attention
and autograd, closed forms, token-permutation invariance, central
differences, and planted slips that must each break a pin."""
import math
import os
import tempfile

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "pooling_oracle.c")


def _problem(seed, n=(5, 0, 9, 1), h=2, S=4, dh=8):
    rng = np.random.default_rng(seed)
    off = np.concatenate([[0], np.cumsum(n)]).astype(np.int64)
    T = int(off[-1])
    f = lambda *s: rng.standard_normal(s).astype(np.float32)   # noqa: E731
    return f(h, S, dh), f(T, h, dh), f(T, h, dh), f(len(n), h, S, dh), off


def _rel(a, b):
    den = max(np.abs(b).max(), 1e-300)
    return float(np.abs(np.asarray(a) - np.asarray(b)).max() / den)


def test_equals_gdpa_with_roles_swapped():
    seeds, k, v, g, off = _problem(1)
    s = 0.4
    o, lse = oracle.pool_fwd(seeds, k, v, off, s)
    ds, dk, dv = oracle.pool_bwd(seeds, k, v, g, off, s)
    h, S, dh = seeds.shape
    q_g = np.ascontiguousarray(seeds.transpose(1, 0, 2))           # S "tokens", h heads
    ds_ref = np.zeros_like(ds)
    for b in range(len(off) - 1):
        t0, t1 = off[b], off[b + 1]
        if t1 == t0:
            assert np.all(o[b] == 0) and np.all(np.isneginf(lse[b]))
            assert np.all(dk[t0:t1] == 0)
            continue
        k_g = np.ascontiguousarray(k[t0:t1].transpose(1, 0, 2))[None]   # [1, h, n_b, dh]
        v_g = np.ascontiguousarray(v[t0:t1].transpose(1, 0, 2))[None]
        og, lg = oracle.fwd(q_g, k_g, v_g, [0, S], "softmax", s)
        assert _rel(o[b], og.transpose(1, 0, 2)) < 1e-13
        assert np.abs(lse[b] - lg).max() < 1e-12
        g_g = np.ascontiguousarray(g[b].transpose(1, 0, 2))
        dqg, dkg, dvg = oracle.bwd(q_g, k_g, v_g, g_g, [0, S], "softmax", s)
        ds_ref += dqg.transpose(1, 0, 2)
        assert _rel(dk[t0:t1], dkg[0].transpose(1, 0, 2)) < 1e-12
        assert _rel(dv[t0:t1], dvg[0].transpose(1, 0, 2)) < 1e-12
    assert _rel(ds, ds_ref) < 1e-12


def test_matches_sdpa_and_autograd():
    seeds, k, v, g, off = _problem(2, n=(7, 3, 12), h=3, S=5, dh=16)
    s = 1 / math.sqrt(16)
    sd = torch.from_numpy(seeds).double().requires_grad_(True)
    kt = torch.from_numpy(k).double().requires_grad_(True)
    vt = torch.from_numpy(v).double().requires_grad_(True)
    outs = []
    for b in range(3):
        t0, t1 = off[b], off[b + 1]
        kb, vb = kt[t0:t1].transpose(0, 1), vt[t0:t1].transpose(0, 1)   # [h, n, dh]
        outs.append(F.scaled_dot_product_attention(sd, kb, vb, scale=s))
    out = torch.stack(outs)
    (out * torch.from_numpy(g).double()).sum().backward()
    o, _ = oracle.pool_fwd(seeds, k, v, off, s)
    assert _rel(o, out.detach().numpy()) < 1e-12
    ds, dk, dv = oracle.pool_bwd(seeds, k, v, g, off, s)
    assert _rel(ds, sd.grad.numpy()) < 1e-12
    assert _rel(dk, kt.grad.numpy()) < 1e-12
    assert _rel(dv, vt.grad.numpy()) < 1e-12


def test_closed_forms():
    seeds, k, v, g, off = _problem(3, n=(1, 6))
    # one token: every seed pools exactly that value row
    o, lse = oracle.pool_fwd(seeds, k, v, off, 0.7)
    np.testing.assert_allclose(o[0], np.broadcast_to(v[0][:, None, :], o[0].shape), atol=1e-15)
    # equal keys within a sample: uniform weights, the mean of the values
    k2 = k.copy()
    k2[1:7] = k2[1]
    o2, lse2 = oracle.pool_fwd(seeds, k2, v, off, 0.7)
    np.testing.assert_allclose(o2[1], np.broadcast_to(v[1:7].astype(np.float64).mean(0)[:, None, :], o2[1].shape),
                               atol=1e-12)
    # ... and LSE = s q.k + ln n
    qk = np.einsum("jsd,jd->js", seeds.astype(np.float64), k2[1].astype(np.float64))
    np.testing.assert_allclose(lse2[1], 0.7 * qk + math.log(6), atol=1e-12)


def test_token_permutation_invariance():
    seeds, k, v, g, off = _problem(4, n=(8, 5))
    perm = np.concatenate([np.random.default_rng(0).permutation(8), 8 + np.arange(5)[::-1]])
    o, _ = oracle.pool_fwd(seeds, k, v, off, 0.5)
    op, _ = oracle.pool_fwd(seeds, k[perm], v[perm], off, 0.5)
    assert _rel(op, o) < 1e-13
    ds, dk, dv = oracle.pool_bwd(seeds, k, v, g, off, 0.5)
    dsp, dkp, dvp = oracle.pool_bwd(seeds, k[perm], v[perm], g, off, 0.5)
    assert _rel(dsp, ds) < 1e-12 and _rel(dkp, dk[perm]) < 1e-12 and _rel(dvp, dv[perm]) < 1e-12


def test_backward_matches_central_differences():
    seeds, k, v, g, off = _problem(5, n=(3, 2), h=2, S=2, dh=3)
    s = 0.6
    ds, dk, dv = oracle.pool_bwd(seeds, k, v, g, off, s)
    gd = g.astype(np.float64)

    def loss(a, b_, c):
        o, _ = oracle.pool_fwd(a.astype(np.float32), b_.astype(np.float32), c.astype(np.float32),
                               off, s)
        return float((o * gd).sum())

    x = [seeds.astype(np.float64), k.astype(np.float64), v.astype(np.float64)]
    eps = 2.0 ** -10
    for idx, grad in enumerate((ds, dk, dv)):
        fd = np.zeros_like(x[idx])
        for i in range(x[idx].size):
            xp, xm = [y.copy() for y in x], [y.copy() for y in x]
            xp[idx].reshape(-1)[i] += eps
            xm[idx].reshape(-1)[i] -= eps
            fd.reshape(-1)[i] = (loss(*xp) - loss(*xm)) / (2 * eps)
        assert _rel(grad, fd) < 2e-5, idx


MUTANTS = {
    "no_scale": ("P[(size_t)i * n + t] = scale * acc;", "P[(size_t)i * n + t] = acc;"),
    "seed_head_offset": ("const float* qb = seeds + (size_t)j * S * dh;\n    const float* kb = k + ((size_t)off[b] * h + j) * dh;\n    const float* vb = v + ((size_t)off[b] * h + j) * dh;\n    probs(S, n, dh, h, qb, kb, scale, P, lb);",
                         "const float* qb = seeds;\n    const float* kb = k + ((size_t)off[b] * h + j) * dh;\n    const float* vb = v + ((size_t)off[b] * h + j) * dh;\n    probs(S, n, dh, h, qb, kb, scale, P, lb);"),
    "dk_no_scale": ("dkb[(size_t)t * h * dh + d] = scale * ak;", "dkb[(size_t)t * h * dh + d] = ak;"),
    "dseeds_last_sample": ("for (int b = 0; b < B; ++b) acc += dq_units", "for (int b = B - 1; b < B; ++b) acc += dq_units"),
    "softmax_grad_sign": ("dA[(size_t)i * n + t] = P[(size_t)i * n + t] * (dA[(size_t)i * n + t] - D);",
                          "dA[(size_t)i * n + t] = P[(size_t)i * n + t] * (dA[(size_t)i * n + t] + D);"),
}
PINS = (test_equals_gdpa_with_roles_swapped, test_matches_sdpa_and_autograd, test_closed_forms)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    with tempfile.TemporaryDirectory() as d:
        msrc = os.path.join(d, "mutant.c")
        open(msrc, "w").write(src.replace(old, new))
        lib = oracle.pool_load(oracle.build(force=True, src=msrc, out=os.path.join(d, "libm.so")))
        saved = oracle._pool_lib
        oracle._pool_lib = lib
        failed = 0
        try:
            for pin in PINS:
                try:
                    pin()
                except AssertionError:
                    failed += 1
        finally:
            oracle._pool_lib = saved
    assert failed, f"mutant {name} passed every pin"
