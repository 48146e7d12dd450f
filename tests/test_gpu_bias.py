"""The biased PFFN variant phi(s Q K^T + b1) V + b2 (gdpa_fwd_bias /
gdpa_bwd_bias) against the fp64 oracle, through the C ABI, element by
element: O, LSE and the gradients dQ, dK, dV, db1, db2, for every phi, head
dim and element type, on jagged cases with empty samples, ragged tails and
key counts that are not multiples of the 128-key block.  Bound: max|gpu -
ref| / max|ref| <= 2e-2 for bf16 inputs (fp32 accumulation), <= 1e-3 for
fp32; the fp32 bias gradients of a bf16 problem sum bf16-rounded dS and take
the bf16 bound."""
import numpy as np
import pytest
import torch

import oracle
import recsys_context_personalised_b200 as pkg
import synthetic as syn

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = {torch.float32: 1e-3, torch.bfloat16: 2e-2}
PHIS = ["identity", "silu", "softmax", "relu", "gelu"]
CASES = [([130, 0, 17, 256], 200), ([1, 127, 128, 129], 128), ([300, 5], 70), ([0, 0], 64)]


def _rel(got, ref):
    got = got.float().cpu().numpy().astype(np.float64)
    if ref.size == 0:
        return 0.0
    den = np.abs(ref).max()
    return float(np.abs(got - ref).max() / den) if den > 0 else float(np.abs(got).max())


def _biases(seed, B, h, m, dh, std=0.5):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(B, h, m, generator=g) * std).float(), \
        (torch.randn(B, h, dh, generator=g) * std).float()


def run_case(n, m, dh, phi, dtype, use_b1=True, use_b2=True, seed=0):
    B, h = len(n), 2
    d = syn.random_problem(200 + seed, B, h, dh, m, n, dtype=dtype, std=0.6)
    b1, b2 = _biases(seed, B, h, m, dh)
    b1 = b1 if use_b1 else None
    b2 = b2 if use_b2 else None
    scale = 1.0 / dh ** 0.5 if phi == "softmax" else 0.5
    q, k, v, g = (d[x].to(DEV) for x in ("q", "k", "v", "dout"))
    off = torch.tensor(d["offsets"], dtype=torch.int32, device=DEV)
    p = pkg.problem_for(q, k, d["offsets"], phi, scale)
    gb1 = b1.to(DEV) if b1 is not None else None
    gb2 = b2.to(DEV) if b2 is not None else None
    o, lse = pkg.fwd_bias(p, q, off, k, v, gb1, gb2)
    dq, dk, dv, db1, db2 = pkg.bwd_bias(p, q, off, k, v, gb1, gb2, o, lse, g)
    torch.cuda.synchronize()
    ro, rl = oracle.fwd(d["q"], d["k"], d["v"], d["offsets"], phi, scale, b1=b1, b2=b2)
    rq, rk, rv, rb1, rb2 = oracle.bwd(d["q"], d["k"], d["v"], d["dout"], d["offsets"], phi, scale,
                                      b1=b1, bias_grads=True)
    tol = TOL[dtype]
    errs = {"o": _rel(o, ro), "dq": _rel(dq, rq), "dk": _rel(dk, rk), "dv": _rel(dv, rv),
            "db1": _rel(db1, rb1), "db2": _rel(db2, rb2)}
    if phi == "softmax" and d["q"].shape[0] > 0:
        errs["lse_abs"] = float(np.abs(lse.cpu().numpy() - rl).max())
    for name, e in errs.items():
        bound = 1e-2 if name == "lse_abs" else tol
        assert e <= bound, f"n={n} m={m} dh={dh} {phi} {dtype}: {name} {e:.3e} > {bound}"
    return errs


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("dh", [32, 64, 128])
@pytest.mark.parametrize("phi", PHIS)
@pytest.mark.parametrize("case", range(len(CASES)))
def test_biased_matches_oracle(case, phi, dh, dtype):
    n, m = CASES[case]
    run_case(n, m, dh, phi, dtype, seed=case)


@pytest.mark.parametrize("phi", ["softmax", "silu"])
@pytest.mark.parametrize("which", ["b1", "b2"])
@pytest.mark.parametrize("dh", [64, 128])
def test_one_bias_only(which, phi, dh):
    run_case([90, 200, 1], 130, dh, phi, torch.bfloat16, use_b1=which == "b1",
             use_b2=which == "b2", seed=7)


@pytest.mark.parametrize("phi", PHIS)
def test_null_biases_equal_the_unbiased_entry_points(phi):
    """gdpa_fwd_bias / gdpa_bwd_bias with NULL biases and NULL bias gradients
    run exactly the kernels of gdpa_fwd / gdpa_bwd."""
    n, m, dh = [130, 17, 256], 200, 64
    d = syn.random_problem(9, 3, 2, dh, m, n, dtype=torch.bfloat16, std=0.6)
    q, k, v, g = (d[x].to(DEV) for x in ("q", "k", "v", "dout"))
    off = torch.tensor(d["offsets"], dtype=torch.int32, device=DEV)
    scale = 0.125 if phi == "softmax" else 0.5
    p = pkg.problem_for(q, k, d["offsets"], phi, scale)
    o1, l1 = pkg.fwd(p, q, off, k, v)
    o2, l2 = pkg.fwd_bias(p, q, off, k, v)
    g1 = pkg.bwd(p, q, off, k, v, o1, l1, g)
    g2 = pkg.bwd_bias(p, q, off, k, v, None, None, o2, l2, g, want_bias_grads=False)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    if phi == "softmax":
        assert torch.equal(l1, l2)
    # dK and dV are summed inside one CTA (deterministic); dQ is reduced in a
    # non-deterministic order, so it matches to rounding only
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
    assert (g1[0].float() - g2[0].float()).abs().max() <= 1e-2 * g1[0].float().abs().max()
    assert g2[3] is None and g2[4] is None
