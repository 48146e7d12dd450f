"""Weight Generation (gdpa_weight_gen: y = ctx w^T rounded to bf16, each
sample's K or V from its context vector) against the fp64 oracle, through the
C ABI.  Bound: max|gpu - ref| / max|ref| <= 2e-2 (bf16 output; the products
run in tf32), element by element, on shapes with ragged sample and feature
tiles, and on the linear-map workload at full size."""
import numpy as np
import pytest
import torch

import oracle
import recsys_context_personalised_b200 as pkg
import synthetic as syn

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = 2e-2


def _rel(got, ref):
    got = got.float().cpu().numpy().astype(np.float64)
    den = np.abs(ref).max()
    return float(np.abs(got - ref).max() / den) if den > 0 else float(np.abs(got).max())


@pytest.mark.parametrize("C", [32, 64])
@pytest.mark.parametrize("B,F", [(1, 8), (5, 136), (128, 1024), (130, 4096), (300, 2056)])
def test_weight_gen_matches_oracle(B, F, C):
    g = torch.Generator().manual_seed(B * 7 + F + C)
    w = torch.randn(F, C, generator=g) / C ** 0.5
    ctx = torch.randn(B, C, generator=g)
    ws = pkg.workspace(256, DEV)
    y = pkg.gdpa.weight_gen(w.to(DEV), ctx.to(DEV), status_ws=ws)
    torch.cuda.synchronize()
    assert pkg.workspace_status(ws) == 0
    err = _rel(y, oracle.weight_gen(w.numpy(), ctx.numpy()))
    assert err <= TOL, err


def test_weight_gen_output_guard():
    """Writes stay inside y: a sentinel-filled buffer around it is untouched."""
    B, F, C = 130, 264, 64
    w, ctx = torch.randn(F, C, device=DEV), torch.randn(B, C, device=DEV)
    big = torch.full(((B + 2) * F,), 3.0, dtype=torch.bfloat16, device=DEV)
    y = big[F:F + B * F].view(B, F)
    pkg.gdpa.weight_gen(w, ctx, y=y)
    torch.cuda.synchronize()
    assert (big[:F] == 3.0).all() and (big[F + B * F:] == 3.0).all()


def test_workload_keys_full_size():
    """The small-m workload's K and V (B = 256, F = h m dh = 65,536, C = 64)
    from the generator's weights and contexts: the GPU map against the
    oracle's on a seeded sample subset, and against the workload's own bf16
    keys (the recipe evaluated in float64) on every sample.  tf32 inputs move
    some outputs across a bf16 rounding boundary, so the comparison is the
    relative measure, not bit equality."""
    wl = syn.WORKLOADS[2]
    full = syn.make_inputs(2)
    for which in ("k", "v"):
        w, ctx = syn.weight_gen_factors(2, which)
        y = pkg.gdpa.weight_gen(w.to(DEV), ctx.to(DEV))
        torch.cuda.synchronize()
        pick = [0, 17, 255]
        ref = oracle.weight_gen(w.numpy(), ctx[pick].numpy())
        assert _rel(y[pick], ref) <= TOL
        recipe = full[which].reshape(wl.B, -1).float()
        dev = (y.cpu().float() - recipe).abs().max() / recipe.abs().max()
        assert dev.item() <= TOL


def _rel64(got, ref):
    got = got.double().cpu().numpy()
    den = np.abs(ref).max()
    return float(np.abs(got - ref).max() / den)


@pytest.mark.parametrize("B,F", [(1, 8), (5, 136), (128, 1024), (130, 4104), (300, 2056),
                                 (896, 512)])
def test_weight_gen_backward_matches_oracle(B, F):
    """dw = dy^T ctx and dctx = dy w (bf16 operands, fp32 accumulation)."""
    C = 64
    g = torch.Generator().manual_seed(B + 3 * F)
    w = torch.randn(F, C, generator=g) / C ** 0.5
    ctx = torch.randn(B, C, generator=g)
    dy = torch.randn(B, F, generator=g).bfloat16()
    dw, dctx = pkg.gdpa.weight_gen_bwd(w.to(DEV), ctx.to(DEV), dy.to(DEV))
    torch.cuda.synchronize()
    rw, rc = oracle.weight_gen_bwd(w.numpy(), ctx.numpy(), dy.float().numpy())
    assert _rel64(dw, rw) <= TOL
    assert _rel64(dctx, rc) <= TOL


def test_weight_gen_backward_two_calls_and_workspace_status():
    """dctx is cleared by every call (not accumulated across calls)."""
    B, F, C = 200, 1032, 64
    w, ctx = torch.randn(F, C, device=DEV), torch.randn(B, C, device=DEV)
    dy = torch.randn(B, F, device=DEV).bfloat16()
    n = ctypes_ws_bytes(B, F, C)
    ws = pkg.workspace(n, DEV)
    a = pkg.gdpa.weight_gen_bwd(w, ctx, dy, ws=ws)
    b = pkg.gdpa.weight_gen_bwd(w, ctx, dy, ws=ws)
    torch.cuda.synchronize()
    assert pkg.workspace_status(ws) == 0
    assert torch.equal(a[0], b[0])
    assert (a[1] - b[1]).abs().max() <= 1e-4 * a[1].abs().max()


def ctypes_ws_bytes(B, F, C):
    import ctypes
    n = ctypes.c_size_t()
    assert pkg.load().gdpa_weight_gen_bwd_workspace_size(B, F, C, ctypes.byref(n)) == 0
    return n.value
