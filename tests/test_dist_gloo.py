"""World-size-2 runs of the benchmark's multi-rank host logic on CPU (gloo).

GDPA's samples are independent, so N ranks run N independent batches with no
collective on the data path; the only collectives are the max-reduction of
the per-rank device times and the sums of work and launches.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        ms = [120.0, 150.0][rank]
        out = bench.aggregate(ms, flops=1e12 * (rank + 1), tokens=1000.0 * (rank + 1),
                              launches=4.0, world=world, dist=dist, device="cpu")
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_aggregate_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=100) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for r in (0, 1):
        o = res[r]
        assert o["ms_max"] == 150.0                      # slowest rank decides
        assert o["flops"] == 3e12 and o["launches"] == 8
        assert o["tflops"] == pytest.approx(3e12 / 0.150 / 1e12)
        assert o["tokens_per_s"] == pytest.approx(3000.0 / 0.150)


def test_aggregate_single_rank_is_identity():
    o = bench.aggregate(200.0, 4e12, 10.0, 3.0, world=1)
    assert o["tflops"] == pytest.approx(20.0) and o["launches"] == 3
