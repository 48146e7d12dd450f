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
