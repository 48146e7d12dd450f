"""Pins of the fp64 GDPA oracle to facts outside itself (CPU only).

Each test checks the oracle against something it does not compute itself:
hand-derived values, closed forms in another association order, library
routines (torch float64 softmax / SiLU / scaled_dot_product_attention /
autograd, scipy logsumexp), invariances of the operator, and central finite
differences of the forward.  A plausible slip in the oracle (a dropped term,
a wrong sign, a transposed operand, a wrong index) breaks at least one of
them; ``test_oracle_mutants`` plants such slips and checks exactly that.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy.special import logsumexp

import oracle
from synthetic import random_problem

HERE = os.path.dirname(os.path.abspath(__file__))
PHIS = ["identity", "silu", "softmax"]
# the PFFN variants' other activations (ReLU, and GELU in its exact form x Phi(x))
PHIS_ALL = PHIS + ["relu", "gelu"]
_LIB_PHI = {"identity": lambda x: x, "silu": F.silu, "softmax": lambda x: torch.softmax(x, dim=-1),
            "relu": F.relu, "gelu": lambda x: F.gelu(x, approximate="none")}


def _f64(x):
    return x.double() if torch.is_tensor(x) else torch.from_numpy(np.asarray(x, np.float64))


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    den = max(np.abs(b).max(), 1e-300)
    return float(np.abs(a - b).max() / den)


def _lib_forward(q, k, v, off, phi, s):
    """Library-routine forward: torch float64 matmul + F.silu / torch.softmax."""
    B, h, m, dh = k.shape
    out = torch.zeros(q.shape, dtype=torch.float64)
    for b in range(B):
        t0, t1 = int(off[b]), int(off[b + 1])
        if t1 == t0:
            continue
        for j in range(h):
            qh = _f64(q[t0:t1, j])
            S = s * (qh @ _f64(k[b, j]).T)
            P = _LIB_PHI[phi](S)
            out[t0:t1, j] = P @ _f64(v[b, j])
    return out.numpy()


def _problem(seed, B=3, h=2, dh=8, m=5, n=(4, 0, 7), std=1.0):
    return random_problem(seed, B, h, dh, m, n, dtype=torch.float32, std=std)


# --------------------------------------------------------------------------
# hand-derived values


@pytest.mark.parametrize("phi", PHIS)
def test_hand_derived_golden(phi):
    g = json.load(open(os.path.join(HERE, "golden", "gdpa_hand_derived.json")))
    inp = g["inputs"]
    q = np.array(inp["q"], np.float32)
    k = np.array(inp["k"], np.float32)
    v = np.array(inp["v"], np.float32)
    dout = np.array(inp["dout"], np.float32)
    off = np.array(inp["offsets"], np.int64)
    want = {key: np.array([eval(e, {"log": math.log}) for e in vals])
            for key, vals in g["cases"][phi].items()}
    scale = eval(inp["scale"], {"log": math.log})
    o, lse = oracle.fwd(q, k, v, off, phi, scale)
    dq, dk, dv = oracle.bwd(q, k, v, dout, off, phi, scale)
    np.testing.assert_allclose(o.reshape(-1), want["o"], rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(dq.reshape(-1), want["dq"], rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(dk.reshape(-1), want["dk"], rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(dv.reshape(-1), want["dv"], rtol=1e-14, atol=1e-14)
    if "lse" in want:
        np.testing.assert_allclose(lse.reshape(-1), want["lse"], rtol=1e-14)


# --------------------------------------------------------------------------
# closed forms and library routines


def test_identity_equals_other_association():
    p = _problem(1, dh=6, m=9, n=(5, 3, 8))
    s = 0.7
    o, _ = oracle.fwd(p["q"], p["k"], p["v"], p["offsets"], "identity", s)
    off = p["offsets"]
    for b in range(3):
        t0, t1 = off[b], off[b + 1]
        for j in range(2):
            Q, K, V = (_f64(p["q"][t0:t1, j]).numpy(), _f64(p["k"][b, j]).numpy(),
                       _f64(p["v"][b, j]).numpy())
            np.testing.assert_allclose(o[t0:t1, j], s * (Q @ (K.T @ V)), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("phi", PHIS_ALL)
def test_matches_library_routines(phi):
    p = _problem(2, B=4, h=3, dh=16, m=11, n=(1, 9, 0, 13))
    s = 0.3 if phi != "softmax" else 0.25
    o, _ = oracle.fwd(p["q"], p["k"], p["v"], p["offsets"], phi, s)
    ref = _lib_forward(p["q"], p["k"], p["v"], p["offsets"], phi, s)
    assert _rel(o, ref) < 1e-12


def test_softmax_matches_sdpa_and_lse():
    p = _problem(3, B=2, h=2, dh=16, m=33, n=(17, 6))
    s = 1.0 / math.sqrt(16)
    o, lse = oracle.fwd(p["q"], p["k"], p["v"], p["offsets"], "softmax", s)
    off = p["offsets"]
    for b in range(2):
        t0, t1 = off[b], off[b + 1]
        for j in range(2):
            qh, kh, vh = _f64(p["q"][t0:t1, j]), _f64(p["k"][b, j]), _f64(p["v"][b, j])
            ref = F.scaled_dot_product_attention(qh[None], kh[None], vh[None], scale=s)[0]
            np.testing.assert_allclose(o[t0:t1, j], ref.numpy(), rtol=1e-12, atol=1e-13)
            S = s * (qh @ kh.T).numpy()
            np.testing.assert_allclose(lse[j, t0:t1], logsumexp(S, axis=1), rtol=1e-13)


def test_softmax_special_cases():
    p = _problem(4, B=2, h=1, dh=8, m=6, n=(5, 4))
    q, k, v, off = p["q"], p["k"].clone(), p["v"].clone(), p["offsets"]
    # all keys equal -> uniform weights -> mean of the value rows
    k_eq = k[:, :, :1].expand_as(k).contiguous()
    o, _ = oracle.fwd(q, k_eq, v, off, "softmax", 0.9)
    for b in range(2):
        np.testing.assert_allclose(o[off[b]:off[b + 1], 0],
                                   np.broadcast_to(_f64(v[b, 0]).mean(0).numpy(), (off[b + 1] - off[b], 8)),
                                   rtol=1e-13, atol=1e-14)
    # all value rows equal -> output equals that row
    v_eq = v[:, :, :1].expand_as(v).contiguous()
    o, _ = oracle.fwd(q, k, v_eq, off, "softmax", 0.9)
    for b in range(2):
        np.testing.assert_allclose(o[off[b]:off[b + 1], 0],
                                   np.broadcast_to(_f64(v[b, 0, 0]).numpy(), (off[b + 1] - off[b], 8)),
                                   rtol=1e-13)
    # zero scale -> mean of the value rows
    o, lse = oracle.fwd(q, k, v, off, "softmax", 0.0)
    for b in range(2):
        np.testing.assert_allclose(o[off[b]:off[b + 1], 0],
                                   np.broadcast_to(_f64(v[b, 0]).mean(0).numpy(), (off[b + 1] - off[b], 8)),
                                   rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, math.log(6), rtol=1e-14)
    # a single key -> that key's value row, LSE = its logit
    o, lse = oracle.fwd(q, k[:, :, :1].contiguous(), v[:, :, :1].contiguous(), off, "softmax", 0.5)
    for b in range(2):
        np.testing.assert_allclose(o[off[b]:off[b + 1], 0],
                                   np.broadcast_to(_f64(v[b, 0, 0]).numpy(), (off[b + 1] - off[b], 8)))


def test_silu_closed_forms():
    # scalar unit: n = m = dh = 1, O = silu(s q k) v
    off = np.array([0, 1], np.int64)
    v = np.array([[[[2.0]]]], np.float32)
    for x, want in [(0.0, 0.0), (math.log(3.0), 0.75 * math.log(3.0)),
                    (-math.log(3.0), -0.25 * math.log(3.0)), (40.0, 40.0), (-40.0, 0.0)]:
        q = np.array([[[1.0]]], np.float32)
        k = np.array([[[[1.0]]]], np.float32)
        o, _ = oracle.fwd(q, k, v, off, "silu", x)
        np.testing.assert_allclose(o[0, 0, 0], 2.0 * want, rtol=1e-15, atol=1e-15)
    # derivative at 0 is one half: dQ = s * (dO . v) * 1/2 * k
    q = np.array([[[0.0]]], np.float32)
    k = np.array([[[[3.0]]]], np.float32)
    g = np.array([[[1.5]]], np.float32)
    dq, dk, dv = oracle.bwd(q, k, v, g, off, "silu", 0.5)
    assert dq[0, 0, 0] == pytest.approx(0.5 * 1.5 * 2.0 * 0.5 * 3.0, rel=1e-15)
    assert dv[0, 0, 0, 0] == 0.0
    # zero keys -> zero output
    p = _problem(5)
    o, _ = oracle.fwd(p["q"], torch.zeros_like(p["k"]), p["v"], p["offsets"], "silu", 1.0)
    assert np.abs(o).max() == 0.0


def test_relu_gelu_closed_forms():
    # one token, three keys with logits S = [1, -1, 1/2] (s = 1, q = e1, k_k = S_k e1),
    # values v = [e1, e2, e1 + e2]:  O = sum_k phi(S_k) v_k
    q = np.array([[[1.0, 0.0]]], np.float32)
    k = np.array([[[[1.0, 0.0], [-1.0, 0.0], [0.5, 0.0]]]], np.float32)
    v = np.array([[[[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]]]], np.float32)
    off = np.array([0, 1], np.int64)
    o, _ = oracle.fwd(q, k, v, off, "relu", 1.0)
    np.testing.assert_allclose(o[0, 0], [1.5, 0.5], rtol=0, atol=1e-15)
    # standard normal CDF from printed tables: Phi(1), Phi(-1), Phi(1/2)
    c1, cm1, ch = 0.8413447460685429, 0.15865525393145707, 0.6914624612740131
    g1, gm1, gh = c1, -cm1, 0.5 * ch
    o, _ = oracle.fwd(q, k, v, off, "gelu", 1.0)
    np.testing.assert_allclose(o[0, 0], [g1 + gh, gm1 + gh], rtol=1e-14)
    # derivatives: ReLU' = [S > 0]; GELU'(x) = Phi(x) + x pdf(x), pdf(1) = pdf(-1) =
    # 0.24197072451914337, pdf(1/2) = 0.3520653267642995 (tables); with dO = e1,
    # dP_k = v_k . e1 = [1, 0, 1] and dV_k = phi(S_k) e1
    dout = np.array([[[1.0, 0.0]]], np.float32)
    dq, dk, dv = oracle.bwd(q, k, v, dout, off, "relu", 1.0)
    np.testing.assert_allclose(dq[0, 0], [1.0 * 1 * 1.0 + 1.0 * 0.5, 0.0], atol=1e-15)
    np.testing.assert_allclose(dv[0, 0, :, 0], [1.0, 0.0, 0.5], atol=1e-15)
    d1, dh_ = c1 + 0.24197072451914337, ch + 0.5 * 0.3520653267642995
    dq, dk, dv = oracle.bwd(q, k, v, dout, off, "gelu", 1.0)
    # dQ = sum_k dS_k k_k with dS = dP * GELU'(S); dK_k = dS_k q
    np.testing.assert_allclose(dq[0, 0, 0], d1 * 1.0 + dh_ * 0.5, rtol=1e-14)
    np.testing.assert_allclose(dk[0, 0, :, 0], [d1, 0.0, dh_], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(dv[0, 0, :, 0], [g1, gm1, gh], rtol=1e-14)


def test_identity_backward_closed_forms():
    p = _problem(6, dh=5, m=7, n=(6, 2, 3))
    s = 1.3
    dq, dk, dv = oracle.bwd(p["q"], p["k"], p["v"], p["dout"], p["offsets"], "identity", s)
    off = p["offsets"]
    for b in range(3):
        t0, t1 = off[b], off[b + 1]
        for j in range(2):
            Q, K, V, G = (_f64(p["q"][t0:t1, j]).numpy(), _f64(p["k"][b, j]).numpy(),
                          _f64(p["v"][b, j]).numpy(), _f64(p["dout"][t0:t1, j]).numpy())
            np.testing.assert_allclose(dv[b, j], s * (K @ (Q.T @ G)), rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(dq[t0:t1, j], s * (G @ (V.T @ K)), rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(dk[b, j], s * (V @ (G.T @ Q)), rtol=1e-12, atol=1e-12)


def test_softmax_backward_invariants():
    p = _problem(7, dh=6, m=9, n=(5, 1, 4))
    s = 0.8
    dq, dk, dv = oracle.bwd(p["q"], p["k"], p["v"], p["dout"], p["offsets"], "softmax", s)
    # shifting all keys of a row by one vector leaves softmax unchanged, so the
    # key gradients of each (sample, head) sum to zero
    assert np.abs(dk.sum(axis=2)).max() < 1e-12
    # equal keys: uniform weights do not depend on q, so dQ is exactly zero
    k_eq = p["k"][:, :, :1].expand_as(p["k"]).contiguous()
    dq, _, _ = oracle.bwd(p["q"], k_eq, p["v"], p["dout"], p["offsets"], "softmax", s)
    assert np.abs(dq).max() < 1e-14


# --------------------------------------------------------------------------
# invariances


@pytest.mark.parametrize("phi", PHIS_ALL)
def test_key_permutation_invariance(phi):
    p = _problem(8, B=2, h=2, dh=4, m=10, n=(6, 3))
    perm = torch.from_numpy(np.random.default_rng(0).permutation(10))
    kp, vp = p["k"][:, :, perm].contiguous(), p["v"][:, :, perm].contiguous()
    o1, l1 = oracle.fwd(p["q"], p["k"], p["v"], p["offsets"], phi, 0.6)
    o2, l2 = oracle.fwd(p["q"], kp, vp, p["offsets"], phi, 0.6)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    g1 = oracle.bwd(p["q"], p["k"], p["v"], p["dout"], p["offsets"], phi, 0.6)
    g2 = oracle.bwd(p["q"], kp, vp, p["dout"], p["offsets"], phi, 0.6)
    np.testing.assert_allclose(g1[0], g2[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(g1[1][:, :, perm.numpy()], g2[1], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(g1[2][:, :, perm.numpy()], g2[2], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("phi", PHIS_ALL)
def test_token_equivariance_and_independence(phi):
    p = _problem(9, B=3, h=2, dh=4, m=6, n=(5, 2, 4))
    off = p["offsets"]
    o, _ = oracle.fwd(p["q"], p["k"], p["v"], off, phi, 0.5)
    # permuting the tokens inside sample 0 permutes its output rows
    perm = np.array([3, 0, 4, 1, 2])
    q2 = p["q"].clone()
    q2[0:5] = p["q"][perm]
    o2, _ = oracle.fwd(q2, p["k"], p["v"], off, phi, 0.5)
    np.testing.assert_allclose(o2[0:5], o[perm], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(o2[5:], o[5:], rtol=0, atol=0)
    # each sample alone gives the same rows as inside the batch
    for b in range(3):
        t0, t1 = off[b], off[b + 1]
        ob, _ = oracle.fwd(p["q"][t0:t1], p["k"][b:b + 1], p["v"][b:b + 1],
                           np.array([0, t1 - t0]), phi, 0.5)
        np.testing.assert_array_equal(ob, o[t0:t1])
    # changing head 1's inputs leaves head 0 untouched
    k3 = p["k"].clone()
    k3[:, 1] *= -2.0
    o3, _ = oracle.fwd(p["q"], k3, p["v"], off, phi, 0.5)
    np.testing.assert_array_equal(o3[:, 0], o[:, 0])
    assert np.abs(o3[:, 1] - o[:, 1]).max() > 0


def test_empty_samples():
    p = _problem(10, B=3, h=2, dh=4, m=5, n=(0, 3, 0))
    o, _ = oracle.fwd(p["q"], p["k"], p["v"], p["offsets"], "softmax", 0.5)
    assert o.shape == (3, 2, 4)
    _, dk, dv = oracle.bwd(p["q"], p["k"], p["v"], p["dout"], p["offsets"], "silu", 0.5)
    assert np.abs(dk[0]).max() == 0 and np.abs(dv[2]).max() == 0
    assert np.abs(dk[1]).max() > 0


def test_bad_arguments_rejected():
    p = _problem(11)
    bad = p["offsets"].copy()
    bad[2] = bad[1] - 1                      # decreasing offsets
    with pytest.raises(RuntimeError):
        oracle.fwd(p["q"], p["k"], p["v"], bad, "silu", 1.0)


# --------------------------------------------------------------------------
# gradients: finite differences (brute force over every input element)


@pytest.mark.parametrize("phi", PHIS_ALL)
def test_backward_matches_central_differences(phi):
    p = random_problem(12, 2, 2, 3, 4, (3, 2), dtype=torch.float32)
    q, k, v, g = (p[x].double().numpy() for x in ("q", "k", "v", "dout"))
    off = p["offsets"]
    s = 0.7

    def loss(qq, kk, vv):
        o, _ = oracle.fwd(qq.astype(np.float32), kk.astype(np.float32),
                          vv.astype(np.float32), off, phi, s)
        return float((o * g).sum())

    # inputs are float32 in the oracle, so perturb by exactly representable steps
    q, k, v = (x.astype(np.float32).astype(np.float64) for x in (q, k, v))
    dq, dk, dv = oracle.bwd(q.astype(np.float32), k.astype(np.float32), v.astype(np.float32),
                            g.astype(np.float32), off, phi, s)
    eps = 2.0 ** -10
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        flat = x.reshape(-1)
        for i in range(flat.size):
            xp, xm = flat.copy(), flat.copy()
            xp[i] += eps
            xm[i] -= eps
            args = {"q": q, "k": k, "v": v}
            args[name] = xp.reshape(x.shape)
            lp = loss(args["q"], args["k"], args["v"])
            args[name] = xm.reshape(x.shape)
            lm = loss(args["q"], args["k"], args["v"])
            fd.reshape(-1)[i] = (lp - lm) / (2 * eps)
        # central differences have O(eps^2) truncation error
        assert _rel(grad, fd) < 2e-5, (name, _rel(grad, fd))


@pytest.mark.parametrize("phi", PHIS_ALL)
def test_backward_matches_torch_autograd(phi):
    p = random_problem(13, 3, 2, 8, 6, (4, 0, 5), dtype=torch.float32)
    off = p["offsets"]
    s = 0.45
    q, k, v = (p[x].double().requires_grad_(True) for x in ("q", "k", "v"))
    g = p["dout"].double()
    out = torch.zeros_like(q)
    outs = []
    for b in range(3):
        t0, t1 = int(off[b]), int(off[b + 1])
        for j in range(2):
            if t1 == t0:
                continue
            S = s * (q[t0:t1, j] @ k[b, j].T)
            P = _LIB_PHI[phi](S)
            outs.append(((t0, t1, j), P @ v[b, j]))
    L = sum((o * g[t0:t1, j]).sum() for (t0, t1, j), o in outs)
    L.backward()
    dq, dk, dv = oracle.bwd(p["q"], p["k"], p["v"], p["dout"], off, phi, s)
    assert _rel(dq, q.grad.numpy()) < 1e-12
    assert _rel(dk, k.grad.numpy()) < 1e-12
    assert _rel(dv, v.grad.numpy()) < 1e-12


# --------------------------------------------------------------------------
# the biased variant phi(s Q K^T + b1) V + b2 (reading R19)


def _biases(seed, B, h, m, dh, scale=1.0):
    rng = np.random.default_rng(seed)
    b1 = (rng.standard_normal((B, h, m)) * scale).astype(np.float32)
    b2 = (rng.standard_normal((B, h, dh)) * scale).astype(np.float32)
    return b1, b2


@pytest.mark.parametrize("phi", PHIS)
def test_bias_hand_derived_golden(phi):
    g = json.load(open(os.path.join(HERE, "golden", "gdpa_bias_hand_derived.json")))
    inp = g["inputs"]
    ev = lambda e: eval(e, {"log": math.log})    # noqa: E731
    q, k, v, dout = (np.array(inp[x], np.float32) for x in ("q", "k", "v", "dout"))
    b1 = np.array([[[ev(e) for e in row] for row in blk] for blk in inp["b1"]], np.float32)
    b2 = np.array([[[ev(e) for e in row] for row in blk] for blk in inp["b2"]], np.float32)
    off = np.array(inp["offsets"], np.int64)
    scale = float(np.float32(ev(inp["scale"])))
    # the exact inputs are fp32 roundings of ln3; the derivation uses ln3 itself
    want = {key: np.array([ev(e) for e in vals]) for key, vals in g["cases"][phi].items()}
    o, lse = oracle.fwd(q, k, v, off, phi, scale, b1=b1, b2=b2)
    dq, dk, dv, db1, db2 = oracle.bwd(q, k, v, dout, off, phi, scale, b1=b1, bias_grads=True)
    got = {"o": o, "dq": dq, "dk": dk, "dv": dv, "db1": db1, "db2": db2, "lse": lse}
    for key, w in want.items():
        np.testing.assert_allclose(got[key].reshape(-1), w, rtol=2e-7, atol=2e-7, err_msg=key)


@pytest.mark.parametrize("phi", PHIS_ALL)
def test_zero_biases_reproduce_the_unbiased_operator(phi):
    p = _problem(31, B=3, h=2, dh=8, m=7, n=(5, 0, 3))
    z1, z2 = np.zeros((3, 2, 7), np.float32), np.zeros((3, 2, 8), np.float32)
    s = 0.6
    a = oracle.fwd(p["q"], p["k"], p["v"], p["offsets"], phi, s)
    b = oracle.fwd(p["q"], p["k"], p["v"], p["offsets"], phi, s, b1=z1, b2=z2)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    ga = oracle.bwd(p["q"], p["k"], p["v"], p["dout"], p["offsets"], phi, s)
    gb = oracle.bwd(p["q"], p["k"], p["v"], p["dout"], p["offsets"], phi, s, b1=z1,
                    bias_grads=True)
    for x, y in zip(ga, gb[:3]):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("phi", PHIS_ALL)
def test_key_bias_is_an_extra_head_dim_column(phi):
    """s (Q K^T) + b1 = s [Q, 1] [K, b1 / s]^T: the unbiased operator on inputs
    with one more head-dim column gives the biased O, dQ, dK, and s * db1 as
    the gradient of that column of K.  s = 1/2 keeps b1 / s exact in fp32."""
    p = _problem(32, B=3, h=2, dh=6, m=5, n=(4, 3, 0))
    s = 0.5
    b1, b2 = _biases(5, 3, 2, 5, 6)
    T = int(p["offsets"][-1])
    qa = np.concatenate([p["q"].numpy(), np.ones((T, 2, 1), np.float32)], -1)
    ka = np.concatenate([p["k"].numpy(), (b1 / s)[..., None]], -1)
    va = np.concatenate([p["v"].numpy(), np.zeros((3, 2, 5, 1), np.float32)], -1)
    ga = np.concatenate([p["dout"].numpy(), np.zeros((T, 2, 1), np.float32)], -1)
    o, lse = oracle.fwd(p["q"], p["k"], p["v"], p["offsets"], phi, s, b1=b1)
    oa, lsea = oracle.fwd(qa, ka, va, p["offsets"], phi, s)
    assert _rel(o, oa[..., :6]) < 1e-13
    if phi == "softmax":
        assert np.abs(lse - lsea).max() < 1e-12
    dq, dk, dv, db1, _ = oracle.bwd(p["q"], p["k"], p["v"], p["dout"], p["offsets"], phi, s,
                                    b1=b1, bias_grads=True)
    dqa, dka, dva = oracle.bwd(qa, ka, va, ga, p["offsets"], phi, s)
    assert _rel(dq, dqa[..., :6]) < 1e-12
    assert _rel(dk, dka[..., :6]) < 1e-12
    assert _rel(dv, dva[..., :6]) < 1e-12
    assert _rel(db1, dka[..., 6] / s) < 1e-12


@pytest.mark.parametrize("phi", PHIS_ALL)
def test_output_bias_shifts_o_and_its_gradient_is_the_token_sum(phi):
    p = _problem(33, B=3, h=2, dh=8, m=6, n=(7, 0, 2))
    s = 0.4
    b1, b2 = _biases(6, 3, 2, 6, 8)
    o1, l1 = oracle.fwd(p["q"], p["k"], p["v"], p["offsets"], phi, s, b1=b1)
    o2, l2 = oracle.fwd(p["q"], p["k"], p["v"], p["offsets"], phi, s, b1=b1, b2=b2)
    off = p["offsets"]
    for b in range(3):
        for j in range(2):
            d = o2[off[b]:off[b + 1], j] - o1[off[b]:off[b + 1], j]
            np.testing.assert_allclose(d, np.broadcast_to(b2[b, j], d.shape), atol=1e-14)
    assert np.array_equal(l1, l2)
    *_, db2 = oracle.bwd(p["q"], p["k"], p["v"], p["dout"], off, phi, s, b1=b1, bias_grads=True)
    g = p["dout"].double().numpy()
    for b in range(3):
        np.testing.assert_allclose(db2[b], g[off[b]:off[b + 1]].sum(0), atol=1e-12)


def test_softmax_key_bias_shift_invariance():
    """Adding c to every key bias of a (sample, head) leaves softmax O, dQ, dK,
    dV and db1 unchanged and moves LSE by c; db1 sums to zero over the keys."""
    p = _problem(34, B=2, h=2, dh=8, m=9, n=(6, 4))
    s = 0.35
    b1, _ = _biases(7, 2, 2, 9, 8)
    b1 = (np.round(b1 * 1024) / 1024).astype(np.float32)    # so that b1 + c is exact in fp32
    c = np.float32(1.25)
    a = oracle.fwd(p["q"], p["k"], p["v"], p["offsets"], "softmax", s, b1=b1)
    b = oracle.fwd(p["q"], p["k"], p["v"], p["offsets"], "softmax", s, b1=b1 + c)
    assert _rel(a[0], b[0]) < 1e-13
    assert np.abs((b[1] - a[1]) - c).max() < 1e-12
    ga = oracle.bwd(p["q"], p["k"], p["v"], p["dout"], p["offsets"], "softmax", s, b1=b1,
                    bias_grads=True)
    gb = oracle.bwd(p["q"], p["k"], p["v"], p["dout"], p["offsets"], "softmax", s, b1=b1 + c,
                    bias_grads=True)
    for x, y in zip(ga, gb):
        assert _rel(x, y) < 1e-11
    assert np.abs(ga[3].sum(-1)).max() < 1e-12


@pytest.mark.parametrize("phi", PHIS_ALL)
def test_biased_operator_matches_torch_autograd(phi):
    p = random_problem(35, 3, 2, 8, 6, (4, 0, 5), dtype=torch.float32)
    off = p["offsets"]
    s = 0.45
    b1n, b2n = _biases(8, 3, 2, 6, 8)
    q, k, v = (p[x].double().requires_grad_(True) for x in ("q", "k", "v"))
    b1 = torch.from_numpy(b1n).double().requires_grad_(True)
    b2 = torch.from_numpy(b2n).double().requires_grad_(True)
    g = p["dout"].double()
    L = 0.0
    ref_o = torch.zeros_like(q)
    for b in range(3):
        t0, t1 = int(off[b]), int(off[b + 1])
        for j in range(2):
            if t1 == t0:
                continue
            x = s * (q[t0:t1, j] @ k[b, j].T) + b1[b, j]
            o = _LIB_PHI[phi](x) @ v[b, j] + b2[b, j]
            ref_o[t0:t1, j] = o.detach()
            L = L + (o * g[t0:t1, j]).sum()
    L.backward()
    o, _ = oracle.fwd(p["q"], p["k"], p["v"], off, phi, s, b1=b1n, b2=b2n)
    assert _rel(o, ref_o.numpy()) < 1e-12
    dq, dk, dv, db1, db2 = oracle.bwd(p["q"], p["k"], p["v"], p["dout"], off, phi, s, b1=b1n,
                                      bias_grads=True)
    for got, ref in ((dq, q.grad), (dk, k.grad), (dv, v.grad), (db1, b1.grad), (db2, b2.grad)):
        assert _rel(got, ref.numpy()) < 1e-12


@pytest.mark.parametrize("phi", PHIS_ALL)
def test_bias_gradients_match_central_differences(phi):
    p = random_problem(36, 2, 2, 3, 4, (3, 2), dtype=torch.float32)
    off = p["offsets"]
    s = 0.7
    g = p["dout"].double().numpy()
    b1, b2 = (x.astype(np.float64) for x in _biases(9, 2, 2, 4, 3, scale=0.5))

    def loss(bb1, bb2):
        o, _ = oracle.fwd(p["q"], p["k"], p["v"], off, phi, s, b1=bb1.astype(np.float32),
                          b2=bb2.astype(np.float32))
        return float((o * g).sum())

    *_, db1, db2 = oracle.bwd(p["q"], p["k"], p["v"], p["dout"], off, phi, s,
                              b1=b1.astype(np.float32), bias_grads=True)
    eps = 2.0 ** -10
    for which, x, grad in (("b1", b1, db1), ("b2", b2, db2)):
        fd = np.zeros_like(x)
        flat = x.reshape(-1)
        for i in range(flat.size):
            xp, xm = flat.copy(), flat.copy()
            xp[i] += eps
            xm[i] -= eps
            if which == "b1":
                lp, lm = loss(xp.reshape(x.shape), b2), loss(xm.reshape(x.shape), b2)
            else:
                lp, lm = loss(b1, xp.reshape(x.shape)), loss(b1, xm.reshape(x.shape))
            fd.reshape(-1)[i] = (lp - lm) / (2 * eps)
        assert _rel(grad, fd) < 2e-5, (which, _rel(grad, fd))
