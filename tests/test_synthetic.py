"""The seeded input generator: determinism, subset consistency, distributions."""
import math

import numpy as np
import torch

import synthetic as syn


def test_splitmix64_matches_python_integer_arithmetic():
    key = syn.stream_key(0, 5, syn.T_Q)
    idx = torch.tensor([0, 1, 2, 12345, 2**40 + 7], dtype=torch.int64)
    got = syn.bits64(key, idx).numpy().astype(np.uint64)
    for i, g in zip(idx.tolist(), got):
        assert int(g) == syn._mix_py(key + (i + 1) * syn._GAMMA)


def test_bf16_rounding_is_round_to_nearest_even():
    x = torch.tensor([1.0 + 2.0**-8, 1.0 + 3 * 2.0**-8, 1.0 + 2.0**-8 + 2.0**-30, -1.0 - 2.0**-8,
                      0.1, -3.3], dtype=torch.float64)
    got = syn.round_to(x, torch.bfloat16).double()
    want = torch.tensor([1.0, 1.0 + 4 * 2.0**-8, 1.0 + 2 * 2.0**-8, -1.0], dtype=torch.float64)
    assert torch.equal(got[:4], want)
    # away from ties the direct rounding agrees with torch's fp32 -> bf16 cast
    assert torch.equal(got[4:], x[4:].float().bfloat16().double())


def test_normal_moments():
    z = syn.normal(syn.stream_key(0, 9, 9), torch.arange(200000)).numpy()
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01


def test_lengths_follow_their_recipes():
    n3 = syn.lengths(syn.WORKLOADS[3])
    assert n3.min() >= 16 and n3.max() <= 2048 and abs(n3.mean() - 1032) < 60
    n4 = syn.lengths(syn.WORKLOADS[4])
    assert n4.min() >= 64 and n4.max() <= 1024
    n5 = syn.lengths(syn.WORKLOADS[5])
    assert n5.min() >= 32 and n5.max() <= 4096
    # truncated power law alpha = 1.5 on [32, 4096]: median ~107, mean ~359
    assert 90 <= np.median(n5) <= 125 and 300 <= n5.mean() <= 420
    assert (syn.lengths(syn.WORKLOADS[2]) == 512).all()


def test_subset_is_bit_identical_to_full_batch():
    full = syn.make_inputs(3, n_override=[5, 0, 9, 3] + [1] * 508)
    sub = syn.make_inputs(3, samples=[2, 0], n_override=[5, 0, 9, 3] + [1] * 508)
    off = full["offsets"]
    assert torch.equal(sub["q"][:9], full["q"][off[2]:off[3]])
    assert torch.equal(sub["q"][9:], full["q"][off[0]:off[1]])
    assert torch.equal(sub["k"][0], full["k"][2]) and torch.equal(sub["v"][1], full["v"][0])


def test_workload_scales():
    d = syn.make_inputs(1)
    assert d["q"].dtype == torch.float32 and abs(d["q"].std().item() - 1 / math.sqrt(32)) < 0.02
    d = syn.make_inputs(2, samples=[0, 1])
    assert d["k"].dtype == torch.bfloat16 and abs(d["k"].float().std().item() - 0.125) < 0.01
    assert abs(d["q"].float().std().item() - 1.0) < 0.02
    d = syn.make_inputs(5, samples=[0])
    assert "dout" in d and abs(d["dout"].float().std().item() - 1.0) < 0.05
