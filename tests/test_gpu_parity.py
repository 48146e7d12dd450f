"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Error measure (the GDPA parity bar): max|gpu - ref| / max|ref| per output
tensor, <= 2e-2 for bf16 inputs with fp32 accumulation and <= 1e-3 for fp32.
Small jagged cases cover every phi and head dim with ragged tails, empty
samples and key counts that are not tile multiples; the five workloads run
at full size in the launch configuration the benchmark times, and are checked
on a seeded subset of samples that the oracle recomputes from inputs it
regenerates on the host.
"""
import numpy as np
import pytest
import torch

import oracle
import recsys_context_personalised_b200 as pkg
import synthetic as syn

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = {torch.float32: 1e-3, torch.bfloat16: 2e-2}


def rel_err(got, ref):
    got = got.float().cpu().numpy().astype(np.float64) if torch.is_tensor(got) else got
    if ref.size == 0:
        return 0.0
    den = np.abs(ref).max()
    return float(np.abs(got - ref).max() / den) if den > 0 else float(np.abs(got).max())


def run_gpu(d, phi, scale, backward, max_n=None):
    q, k, v = (d[x].to(DEV) for x in ("q", "k", "v"))
    off = torch.tensor(d["offsets"], dtype=torch.int32, device=DEV)
    p = pkg.problem_for(q, k, d["offsets"], phi, scale, max_n=max_n)
    o, lse = pkg.fwd(p, q, off, k, v)
    out = {"o": o, "lse": lse}
    if backward:
        g = d["dout"].to(DEV)
        out["dq"], out["dk"], out["dv"] = pkg.bwd(p, q, off, k, v, o, lse, g)
    torch.cuda.synchronize()
    return out


def check(out, d, phi, scale, backward, dtype, label=""):
    ro, rl = oracle.fwd(d["q"], d["k"], d["v"], d["offsets"], phi, scale)
    tol = TOL[dtype]
    errs = {"o": rel_err(out["o"], ro)}
    if phi == "softmax" and d["q"].shape[0] > 0:
        errs["lse_abs"] = float(np.abs(out["lse"].cpu().numpy() - rl).max())
    if backward:
        rq, rk, rv = oracle.bwd(d["q"], d["k"], d["v"], d["dout"], d["offsets"], phi, scale)
        errs.update(dq=rel_err(out["dq"], rq), dk=rel_err(out["dk"], rk), dv=rel_err(out["dv"], rv))
    for name, e in errs.items():
        bound = 1e-2 if name == "lse_abs" else tol
        assert e <= bound, f"{label} {name}: {e:.3e} > {bound}"
    return errs


# identity, SiLU, softmax and the PFFN variants' other activations
PHIS = ["identity", "silu", "softmax", "relu", "gelu"]

SMALL = [
    # (n per sample, m)
    ([130, 0, 17, 256], 200),
    ([1, 127, 128, 129], 128),
    ([300, 5], 1),
    ([64, 64, 64], 130),
    ([0, 0, 3], 257),
    ([513], 64),
    ([0, 0], 64),          # no tokens at all: dK = dV = 0
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("dh", [32, 64, 128])
@pytest.mark.parametrize("phi", PHIS)
@pytest.mark.parametrize("case", range(len(SMALL)))
def test_small_jagged(case, phi, dh, dtype):
    n, m = SMALL[case]
    d = syn.random_problem(100 + case, len(n), 2, dh, m, n, dtype=dtype, std=0.6)
    scale = 1.0 / dh ** 0.5 if phi == "softmax" else 0.5
    out = run_gpu(d, phi, scale, True)
    if phi == "softmax" and m == 1:
        check_single_key_softmax(out, d, scale, TOL[dtype])
        return
    check(out, d, phi, scale, True, dtype, f"n={n} m={m}")


@pytest.mark.parametrize("phi", PHIS)
@pytest.mark.parametrize("n", [[100], [300, 7], [129, 0, 640]])
def test_odd_head_count(n, phi):
    """h = 3: the work list can hold an odd number of tiles and mixes tiles of
    different (sample, head) in one CTA work item."""
    d = syn.random_problem(21, len(n), 3, 64, 300, n, dtype=torch.bfloat16, std=0.6)
    scale = 0.125 if phi == "softmax" else 0.5
    out = run_gpu(d, phi, scale, True)
    check(out, d, phi, scale, True, torch.bfloat16, f"h=3 n={n}")


@pytest.mark.parametrize("phi", ["softmax", "silu"])
@pytest.mark.parametrize("dh", [64, 128])
def test_many_samples_unsorted_work_list(phi, dh):
    """B = 4500 > 4096: the backward's work list is not sorted by length, and
    thousands of one-tile items, a third of them without tokens, pass through
    each CTA's K/V slots, staging buffers and statistics ring."""
    rng = np.random.default_rng(7)
    n = rng.choice([0, 1, 2, 50, 130], size=4500, p=[0.3, 0.2, 0.2, 0.2, 0.1]).tolist()
    d = syn.random_problem(61, len(n), 2, dh, 64, n, dtype=torch.bfloat16, std=0.6)
    scale = 1.0 / dh ** 0.5 if phi == "softmax" else 0.5
    out = run_gpu(d, phi, scale, True)
    check(out, d, phi, scale, True, torch.bfloat16, f"B=4500 dh={dh}")


@pytest.mark.parametrize("dh", [32, 64, 128])
def test_softmax_row_max_growth(dh):
    """Logits that grow from one key block to the next (and one that jumps by
    far more than 2^8 in log2 units) exercise the exact-max fallback and the
    O rescaling of the online softmax."""
    n, m = [200, 77], 640
    d = syn.random_problem(31, len(n), 2, dh, m, n, dtype=torch.bfloat16, std=0.5)
    growth = torch.ones(m)
    for j in range(5):
        growth[128 * j:128 * (j + 1)] = 1.0 + 1.5 * j
    growth[600:] = 12.0
    d["k"] = (d["k"].float() * growth[None, None, :, None]).bfloat16()
    scale = 1.0 / dh ** 0.5
    out = run_gpu(d, "softmax", scale, True)
    check(out, d, "softmax", scale, True, torch.bfloat16, f"growth dh={dh}")


@pytest.mark.parametrize("phi", PHIS)
def test_negative_scale(phi):
    """A negative scale flips the logits (the softmax kernels then track a row
    minimum of the raw dot products)."""
    n, m = [150, 33], 300
    d = syn.random_problem(41, len(n), 2, 64, m, n, dtype=torch.bfloat16, std=0.6)
    out = run_gpu(d, phi, -0.3, True)
    check(out, d, phi, -0.3, True, torch.bfloat16, "negative scale")


def test_bounded_wait_times_out_and_context_survives():
    """A device wait that can never complete gives up after its limit, reports
    GDPA_ERR_TIMEOUT through the workspace status word, and later work runs."""
    import ctypes
    lib = pkg.load()
    lib.gdpa_selftest_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint32,
                                               ctypes.c_void_p]
    lib.gdpa_selftest_wait_timeout.restype = ctypes.c_int
    ws = pkg.workspace(256, DEV)
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.gdpa_selftest_wait_timeout(ws.data_ptr(), ws.numel(), 20000, stream) == 0
    assert pkg.workspace_status(ws) == 4
    d = syn.random_problem(5, 2, 2, 64, 64, [10, 20], dtype=torch.bfloat16)
    out = run_gpu(d, "silu", 0.5, False)
    check(out, d, "silu", 0.5, False, torch.bfloat16, "after time-out")


def check_single_key_softmax(out, d, scale, tol):
    """Softmax over one key: P = 1, so dS = dP - D = 0 and dQ = dK = 0 exactly.

    The relative measure is undefined for an all-zero reference; the GPU's
    residual comes from D = rowsum(dO * O) taken on the rounded O.  It is
    bounded here by `tol` times the size of the terms that cancel,
    scale * max|dP| * max|K| (dQ) and scale * max|dP| * max|Q| (dK).
    """
    ro, _ = oracle.fwd(d["q"], d["k"], d["v"], d["offsets"], "softmax", scale)
    rq, rk, rv = oracle.bwd(d["q"], d["k"], d["v"], d["dout"], d["offsets"], "softmax", scale)
    assert rel_err(out["o"], ro) <= tol and rel_err(out["dv"], rv) <= tol
    g, v = d["dout"].double().numpy(), d["v"].double().numpy()
    dp = np.abs(np.einsum("thd,bhmd->thm", g, v)).max() if g.size else 0.0
    kmax, qmax = float(d["k"].abs().max()), float(d["q"].abs().max()) if g.size else 0.0
    assert np.abs(out["dq"].float().cpu().numpy()).max(initial=0.0) <= tol * scale * dp * kmax
    assert np.abs(out["dk"].float().cpu().numpy()).max(initial=0.0) <= tol * scale * dp * qmax


@pytest.mark.parametrize("dh", [64, 128])
@pytest.mark.parametrize("phi", ["softmax", "silu"])
def test_outputs_untouched_outside_their_ranges(phi, dh):
    """Guard regions around every output of the forward and the backward.

    o, lse and dq sit 64 rows (lse: 64 values) into larger sentinel-filled
    buffers, dk and dv one sample in, and the workspaces are 4 KB longer than
    asked for.  Ragged lengths and m = 70 (not a multiple of the 128-key
    block) put partial tiles at both ends.  Every sentinel before and after
    each output must be untouched, and the outputs inside must still match
    the oracle.
    """
    n, m, h = [129, 3, 0, 200], 70, 2
    B = len(n)
    d = syn.random_problem(7, B, h, dh, m, n, dtype=torch.bfloat16, std=0.6)
    q, k, v, g = (d[x].to(DEV) for x in ("q", "k", "v", "dout"))
    off = torch.tensor(d["offsets"], dtype=torch.int32, device=DEV)
    T = int(d["offsets"][-1])
    scale = 1.0 / dh ** 0.5 if phi == "softmax" else 0.5
    p = pkg.problem_for(q, k, d["offsets"], phi, scale)
    bf = torch.bfloat16
    o_big = torch.full((T + 128, h, dh), 7.0, dtype=bf, device=DEV)
    dq_big = torch.full((T + 128, h, dh), 5.0, dtype=bf, device=DEV)
    dk_big = torch.full((B + 2, h, m, dh), 9.0, dtype=bf, device=DEV)
    dv_big = torch.full((B + 2, h, m, dh), 11.0, dtype=bf, device=DEV)
    lse_big = torch.full((h * T + 128,), 3.0, dtype=torch.float32, device=DEV)
    o, dq = o_big[64:64 + T], dq_big[64:64 + T]
    dk, dv = dk_big[1:B + 1], dv_big[1:B + 1]
    lse = lse_big[64:64 + h * T].view(h, T)
    nf, nb = pkg.fwd_workspace_bytes(p), pkg.bwd_workspace_bytes(p)
    wsf = torch.full((nf + 4096,), 0xAB, dtype=torch.uint8, device=DEV)
    wsb = torch.full((nb + 4096,), 0xAB, dtype=torch.uint8, device=DEV)
    pkg.fwd(p, q, off, k, v, o=o, lse=lse, ws=wsf)
    pkg.bwd(p, q, off, k, v, o, lse, g, dq=dq, dk=dk, dv=dv, ws=wsb)
    torch.cuda.synchronize()
    assert pkg.workspace_status(wsf) == 0 and pkg.workspace_status(wsb) == 0
    for name, big, lo, hi, val in (("o", o_big, 64, 64 + T, 7.0), ("dq", dq_big, 64, 64 + T, 5.0),
                                   ("dk", dk_big, 1, B + 1, 9.0), ("dv", dv_big, 1, B + 1, 11.0),
                                   ("lse", lse_big, 64, 64 + h * T, 3.0)):
        assert (big[:lo] == val).all(), f"{name}: written before its range"
        assert (big[hi:] == val).all(), f"{name}: written past its range"
    assert (wsf[nf:] == 0xAB).all() and (wsb[nb:] == 0xAB).all(), "workspace overrun"
    out = {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}
    check(out, d, phi, scale, True, torch.bfloat16, f"guarded {phi} dh={dh}")


def test_bad_device_offsets_reported_not_crashing():
    d = syn.random_problem(3, 3, 2, 64, 64, [10, 20, 30], dtype=torch.bfloat16)
    q, k, v = (d[x].to(DEV) for x in ("q", "k", "v"))
    bad = torch.tensor([0, 25, 20, 60], dtype=torch.int32, device=DEV)   # decreasing
    p = pkg.problem_for(q, k, d["offsets"], "silu", 1.0)
    ws = pkg.workspace(pkg.fwd_workspace_bytes(p), DEV)
    pkg.fwd(p, q, bad, k, v, ws=ws)
    assert pkg.workspace_status(ws) == 1
    good = torch.tensor(d["offsets"], dtype=torch.int32, device=DEV)
    pkg.fwd(p, q, good, k, v, ws=ws)
    assert pkg.workspace_status(ws) == 0


def _subset(wl, n, rng_seed=0, count=3):
    rng = np.random.default_rng(rng_seed)
    picks = {int(np.argmax(n)), int(np.argmin(n))}
    picks |= set(int(x) for x in rng.choice(len(n), size=count, replace=False))
    return sorted(picks)


@pytest.mark.parametrize("wid", [1, 2, 3, 4, 5])
def test_workload_full_size(wid):
    wl = syn.WORKLOADS[wid]
    full = syn.make_inputs(wid, device=DEV, backward=True)
    out = run_gpu(full, wl.phi_name, wl.scale, True, max_n=int(full["lengths"].max()))
    samples = list(range(wl.B)) if wid == 1 else _subset(wl, full["lengths"])
    sub = syn.make_inputs(wid, device="cpu", samples=samples, backward=True)
    off = full["offsets"]
    rows = np.concatenate([np.arange(off[b], off[b + 1]) for b in samples])
    rows_t = torch.from_numpy(rows).to(DEV)
    sel = torch.tensor(samples, device=DEV)
    got = {"o": out["o"][rows_t], "dq": out["dq"][rows_t], "dk": out["dk"][sel],
           "dv": out["dv"][sel]}
    if out["lse"] is not None:
        got["lse"] = out["lse"][:, rows_t]
    # the device-generated inputs of the checked samples equal the host ones
    # (one bf16 ulp at a rare rounding tie is the most a host/device libm
    # difference can change; the oracle always reads the host copy)
    for a, b in ((full["q"][rows_t].cpu(), sub["q"]), (full["k"][sel].cpu(), sub["k"]),
                 (full["v"][sel].cpu(), sub["v"])):
        diff = (a.float() - b.float()).abs()
        assert (diff > 0).float().mean().item() < 1e-5
        assert diff.max().item() <= 2.0 ** -6 * b.float().abs().max().item()
    errs = check(got, sub, wl.phi_name, wl.scale, True, wl.dtype, wl.name)
    print(wl.name, samples, errs)
