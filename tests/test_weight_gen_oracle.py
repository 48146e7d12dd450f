"""Pins of the fp64 Weight Generation oracle (Y = ctx W^T: each sample's K or
V generated from its context vector) to facts outside itself, CPU only:
hand-derived values, one-hot contexts, linearity, a library matmul, torch
autograd, central differences, the workload recipe the input generator
states, and planted slips that each break at least one pin."""
import os
import tempfile

import numpy as np
import pytest
import torch

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "weight_gen_oracle.c")


def _rand(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape).astype(np.float32)


def test_hand_derived():
    # W = [[1, 2], [3, 4], [5, 6]], ctx = [[1, -1]]: Y = [1-2, 3-4, 5-6] = [-1, -1, -1];
    # dY = [[1, 0, 2]]: dW = dY^T ctx = [[1, -1], [0, 0], [2, -2]],
    # dctx = dY W = [1 + 10, 2 + 12] = [11, 14]
    w = np.array([[1, 2], [3, 4], [5, 6]], np.float32)
    c = np.array([[1, -1]], np.float32)
    np.testing.assert_array_equal(oracle.weight_gen(w, c), [[-1, -1, -1]])
    dw, dc = oracle.weight_gen_bwd(w, c, np.array([[1, 0, 2]], np.float32))
    np.testing.assert_array_equal(dw, [[1, -1], [0, 0], [2, -2]])
    np.testing.assert_array_equal(dc, [[11, 14]])


def test_one_hot_context_selects_a_column():
    w = _rand(1, 37, 8)
    ctx = np.eye(8, dtype=np.float32)
    y = oracle.weight_gen(w, ctx)
    np.testing.assert_array_equal(y, w.T.astype(np.float64))


def test_linear_in_the_context():
    w = _rand(2, 50, 16)
    # contexts on a 2^-8 grid: 2 c1 - 0.5 c2 is then exact in fp32
    c1, c2 = (np.round(_rand(s, 4, 16) * 256) / 256 for s in (3, 4))
    y = oracle.weight_gen(w, (2 * c1 - 0.5 * c2).astype(np.float32))
    y12 = 2 * oracle.weight_gen(w, c1.astype(np.float32)) - \
        0.5 * oracle.weight_gen(w, c2.astype(np.float32))
    assert np.abs(y - y12).max() <= 1e-12 * np.abs(y).max()


def test_matches_library_matmul():
    w, c = _rand(5, 300, 64), _rand(6, 9, 64)
    ref = torch.from_numpy(c).double() @ torch.from_numpy(w).double().T
    assert np.abs(oracle.weight_gen(w, c) - ref.numpy()).max() <= 1e-12 * np.abs(ref.numpy()).max()


def test_backward_matches_torch_autograd():
    w0, c0, g = _rand(7, 40, 12), _rand(8, 5, 12), _rand(9, 5, 40)
    w = torch.from_numpy(w0).double().requires_grad_(True)
    c = torch.from_numpy(c0).double().requires_grad_(True)
    ((c @ w.T) * torch.from_numpy(g).double()).sum().backward()
    dw, dc = oracle.weight_gen_bwd(w0, c0, g)
    assert np.abs(dw - w.grad.numpy()).max() <= 1e-12 * np.abs(dw).max()
    assert np.abs(dc - c.grad.numpy()).max() <= 1e-12 * np.abs(dc).max()


def test_backward_matches_central_differences():
    w, c, g = (x.astype(np.float64) for x in (_rand(10, 6, 3), _rand(11, 2, 3), _rand(12, 2, 6)))

    def loss(ww, cc):
        return float((oracle.weight_gen(ww.astype(np.float32), cc.astype(np.float32)) * g).sum())

    dw, dc = oracle.weight_gen_bwd(w.astype(np.float32), c.astype(np.float32), g.astype(np.float32))
    eps = 2.0 ** -10
    for which, x, grad in (("w", w, dw), ("c", c, dc)):
        fd = np.zeros_like(x)
        for i in range(x.size):
            xp, xm = x.copy().reshape(-1), x.copy().reshape(-1)
            xp[i] += eps
            xm[i] -= eps
            if which == "w":
                fd.reshape(-1)[i] = (loss(xp.reshape(x.shape), c) - loss(xm.reshape(x.shape), c)) / (2 * eps)
            else:
                fd.reshape(-1)[i] = (loss(w, xp.reshape(x.shape)) - loss(w, xm.reshape(x.shape))) / (2 * eps)
        # the loss is linear in each argument: central differences are exact up to rounding
        assert np.abs(grad - fd).max() <= 1e-9 * max(np.abs(fd).max(), 1.0), which


def test_workload_recipe_keys_are_the_oracle_map():
    """The bf16 keys of the small-m workload (a random linear map of a 64-dim
    context, as the workload text states) are the oracle's map of the same
    weight and contexts, rounded once to bf16."""
    import synthetic as syn
    samples = [0, 5, 255]
    d = syn.make_inputs(2, samples=samples)
    w, ctx = syn.weight_gen_factors(2, "k", samples=samples)
    y = oracle.weight_gen(w, ctx)
    k_ref = syn.round_to(torch.from_numpy(y), torch.bfloat16).float().numpy()
    k = d["k"].float().numpy().reshape(len(samples), -1)
    assert (k != k_ref).mean() < 1e-5


MUTANTS = {
    "w_transposed": ("acc += (double)W[f * C + c] * (double)ctx[(int64_t)b * C + c];",
                     "acc += (double)W[c * F + f] * (double)ctx[(int64_t)b * C + c];"),
    "ctx_first_sample": ("acc += (double)W[f * C + c] * (double)ctx[(int64_t)b * C + c];",
                         "acc += (double)W[f * C + c] * (double)ctx[c];"),
    "dw_uses_w": ("acc += (double)dy[(int64_t)b * F + f] * (double)ctx[(int64_t)b * C + c];",
                  "acc += (double)dy[(int64_t)b * F + f] * (double)W[f * C + c];"),
    "dctx_uses_ctx": ("acc += (double)dy[(int64_t)b * F + f] * (double)W[f * C + c];",
                      "acc += (double)dy[(int64_t)b * F + f] * (double)ctx[(int64_t)b * C + c];"),
}
PINS = (test_hand_derived, test_one_hot_context_selects_a_column, test_matches_library_matmul,
        test_backward_matches_torch_autograd)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    with tempfile.TemporaryDirectory() as d:
        msrc = os.path.join(d, "mutant.c")
        open(msrc, "w").write(src.replace(old, new))
        lib = oracle.wg_load(oracle.build(force=True, src=msrc, out=os.path.join(d, "libm.so")))
        saved = oracle._wg_lib
        oracle._wg_lib = lib
        failed = 0
        try:
            for pin in PINS:
                try:
                    pin()
                except AssertionError:
                    failed += 1
        finally:
            oracle._wg_lib = saved
    assert failed, f"mutant {name} passed every pin"
