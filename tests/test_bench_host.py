"""Host logic of bench.py that needs no GPU: workload selection, the --phi
override, the end-to-end chunking, the oracle sample, the peak choice, the
traffic record's source hash and the multi-rank launch."""
import argparse

import numpy as np
import os

import pytest

import bench
import synthetic as syn


def _ns(**kw):
    base = dict(phi=None, workload=bench.DEFAULT_WORKLOAD)
    base.update(kw)
    return argparse.Namespace(**base)


def test_default_workload_is_the_softmax_fwd_bwd_one():
    wl = bench.workload(_ns())
    assert wl is syn.WORKLOADS[5]
    assert wl.phi_name == "softmax" and wl.backward
    assert bench.metric_name(wl) == "GDPA fwd+bwd TFLOP/s"
    assert bench.parse([]).workload == 5


@pytest.mark.parametrize("wid", [1, 2, 3, 4, 5])
def test_workload_option_selects_each_shape(wid):
    args = bench.parse(["--workload", str(wid)])
    wl = bench.workload(args)
    assert wl is syn.WORKLOADS[wid]
    assert bench.step_flop_units(wl) == (12 if wl.backward else 4)
    assert bench.metric_name(wl).startswith("GDPA fwd+bwd" if wl.backward else "GDPA fwd ")


def test_forward_bytes_of_the_small_m_workload():
    wl = syn.WORKLOADS[2]
    T = 256 * 512
    # Q and O: T*h*dh bf16 each; K and V: B*h*m*dh bf16 each; no LSE for SiLU
    assert bench.fwd_bytes(wl, T) == 2 * (2 * T * 4 * 64 + 2 * 256 * 4 * 256 * 64)
    wl5 = syn.WORKLOADS[5]
    assert bench.fwd_bytes(wl5, 10) == 2 * (2 * 10 * 16 * 64 + 2 * 1024 * 16 * 2048 * 64) + \
        4 * 10 * 16


def test_phi_override_keeps_shapes_and_scale():
    base = syn.WORKLOADS[bench.DEFAULT_WORKLOAD]
    for phi in ("relu", "gelu", "silu", "identity"):
        wl = bench.workload(_ns(phi=phi))
        assert wl.phi_name == phi
        assert phi in wl.name and "softmax" not in wl.name
        assert (wl.B, wl.h, wl.dh, wl.m, wl.scale, wl.lengths) == \
            (base.B, base.h, base.dh, base.m, base.scale, base.lengths)
    assert bench.workload(_ns(phi="softmax")) is base


def test_e2e_chunks_cover_every_sample_once():
    import numpy as np
    for B, nchunks in ((1024, 8), (5, 8), (7, 3), (1, 1)):
        n = np.random.default_rng(B).integers(0, 50, size=B)
        off = [0] + np.cumsum(n).tolist()
        ch = bench.e2e_chunks(off, nchunks)
        assert ch[0][0][0] == 0 and ch[-1][0][1] == B
        assert all(b1 > b0 for (b0, b1), _ in ch)
        for ((_, e0), (_, r0)), ((s1, _), (t1, _)) in zip(ch, ch[1:]):
            assert e0 == s1 and r0 == t1                      # contiguous samples and rows
        assert all(t0 == off[b0] and t1 == off[b1] for (b0, b1), (t0, t1) in ch)
        assert len(ch) == min(nchunks, B)


@pytest.mark.parametrize("wid", [1, 3, 5])
def test_oracle_sample_is_fixed_and_bounded(wid):
    """Both oracle legs (cpu_baseline and --impl reference) time the same samples."""
    wl = syn.WORKLOADS[wid]
    n = syn.lengths(wl)
    a, b = bench.oracle_sample(wl, n), bench.oracle_sample(wl, n)
    assert a == b and a == sorted(set(a)) and len(a) >= 1
    flops = sum(bench._oracle_unit_flops(n[i], wl) for i in a)
    assert flops <= bench.ORACLE_STEP_FLOPS or len(a) == 1


def test_config_identical_in_both_arms():
    wl = syn.WORKLOADS[5]
    T = int(syn.lengths(wl).sum())
    assert bench.config_dict(wl, T, 1) == bench.config_dict(wl, T, 1)
    assert bench.config_dict(wl, T, 1)["tokens_per_rank"] == T


def test_peak_choice_follows_the_clock():
    pk = dict(hbm=6500.0, bf16=1643.0, bf16_sustained=1365.0, source="measured",
              sustained_mhz=1305.0)
    v, why = bench.choose_bf16_peak(pk, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0})
    assert v == 1643.0 and "burst" in why
    v, why = bench.choose_bf16_peak(pk, {"sm_mhz": 1300.0, "sm_max_mhz": 1965.0})
    assert v == 1365.0 and "sustained" in why
    v, _ = bench.choose_bf16_peak(pk, None)
    assert v == 1643.0


def test_traffic_record_goes_null_when_the_kernel_source_changes(monkeypatch):
    sha = bench.sources_sha16("gdpa_fwd_sm100")
    assert len(sha) == 16
    monkeypatch.setattr(bench, "TRAFFIC_PER_UNIT", {"gdpa_fwd_sm100": {5: (2.0, sha)}})
    assert bench.traffic_for("gdpa_fwd_sm100", 5, 10.0) == 20.0
    assert bench.traffic_for("gdpa_fwd_sm100", 3, 10.0) is None
    monkeypatch.setattr(bench, "TRAFFIC_PER_UNIT", {"gdpa_fwd_sm100": {5: (2.0, "0" * 16)}})
    assert bench.traffic_for("gdpa_fwd_sm100", 5, 10.0) is None


def test_recorded_traffic_entries_name_known_kernels():
    for kern, per_wl in bench.TRAFFIC_PER_UNIT.items():
        assert kern in bench.KERNEL_SOURCES
        for wid, (bpu, sha) in per_wl.items():
            assert wid in syn.WORKLOADS and bpu > 0 and len(sha) == 16


def test_gpus_without_torchrun_relaunches_under_torchrun():
    cmd = bench.torchrun_command(["--gpus", "4", "--steps", "2"], 4, 29500)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert cmd[-3:] == ["--gpus", "4", "--steps", "2"] or cmd[-4:] == ["--gpus", "4", "--steps", "2"]
    assert os.path.basename(cmd[cmd.index("--master-port=29500") + 1]) == "bench.py"


def test_world_size_must_match_gpus(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert bench.world_from_env(bench.parse(["--gpus", "2"])) == (1, 2, 1)
    with pytest.raises(SystemExit):
        bench.world_from_env(bench.parse(["--gpus", "4"]))


def test_variant_flops_window_counts_the_keys_of_every_window():
    """4*h*dh per (query, key) pair of the causal window t - W < t' <= t,
    counted one token at a time."""
    rng = np.random.default_rng(3)
    lengths = rng.integers(0, 700, size=40)
    for W in (1, 2, 17, 128, 1000):
        pairs = sum(min(W, t + 1) for n in lengths for t in range(int(n)))
        assert bench.variant_flops("window", lengths, 16, 64, window=W) == 4.0 * 16 * 64 * pairs


def test_variant_flops_pool_is_seeds_times_tokens():
    lengths = [0, 5, 130]
    assert bench.variant_flops("pool", lengths, 16, 64, S=64) == 4.0 * 64 * 135 * 16 * 64


def test_variant_oracle_sample_fills_its_budget_and_is_fixed():
    lengths = np.arange(1, 200)
    f = lambda n: float(sum(n))
    a = bench.variant_oracle_sample(lengths, f, budget=500.0)
    assert a == bench.variant_oracle_sample(lengths, f, budget=500.0)
    assert a == sorted(set(a)) and sum(lengths[b] for b in a) <= 500 + max(lengths)


def test_pool_and_window_are_exclusive():
    with pytest.raises(SystemExit):
        bench.main(["--pool", "64", "--window", "128"])
