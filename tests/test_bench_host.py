"""Host logic of bench.py that needs no GPU: the --phi workload override."""
import argparse

import bench
import synthetic as syn


def test_default_workload_is_the_softmax_fwd_bwd_one():
    wl = bench.workload(argparse.Namespace(phi=None))
    assert wl is syn.WORKLOADS[bench.WORKLOAD]
    assert wl.phi_name == "softmax" and wl.backward


def test_phi_override_keeps_shapes_and_scale():
    base = syn.WORKLOADS[bench.WORKLOAD]
    for phi in ("relu", "gelu", "silu", "identity"):
        wl = bench.workload(argparse.Namespace(phi=phi))
        assert wl.phi_name == phi
        assert phi in wl.name and "softmax" not in wl.name
        assert (wl.B, wl.h, wl.dh, wl.m, wl.scale, wl.lengths) == \
            (base.B, base.h, base.dh, base.m, base.scale, base.lengths)
    assert bench.workload(argparse.Namespace(phi="softmax")) is base
