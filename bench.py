#!/usr/bin/env python
"""GDPA benchmark: TFLOP/s of the fused hot path on one B200 (or N replicas).

One step = the whole GDPA hot path over one synthetic batch: tile scheduling,
the fused forward (S = s Q K^T, P = phi(S), O = P V, softmax statistics) and,
for the workloads that train (4 and 5), the fused backward (dQ, dK, dV).  The
default workload is the largest jagged bf16 softmax problem: B = 1024 samples
with power-law (alpha = 1.5) history lengths on [32, 4096], h = 16 heads,
dh = 64, m = 2048 context keys per sample and head, scale 1/sqrt(dh).
``--workload 1..5`` runs any of the five problem shapes.

Throughput counts algorithmic FLOPs only: forward 4*T*h*m*dh, backward
8*T*h*m*dh (the recomputation of S in the backward is not credited).  Every
step is bracketed by its own CUDA events, and the L2 is flushed (a 256 MB
write) between steps, outside the events.

Multi-GPU: samples are independent and the op has no exchange step, so N
ranks run N independent batches (weak scaling, no collective on the data
path; a barrier and one max-reduction of the timings only).  ``--gpus N``
without a torchrun environment relaunches itself under torchrun.

``--impl reference`` times the fp64 CPU oracle on a fixed seeded sample of
the same workload (rank 0 only), in the same units.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import socket
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)
CSRC = os.path.join(ROOT, "recsys_context_personalised_b200", "csrc")

DEFAULT_WORKLOAD = 5
E2E_CHUNKS = 8                          # sample groups of the end-to-end step
FLOPS_FWD, FLOPS_BWD = 4, 8            # x T*h*m*dh
L2_FLUSH_BYTES = 256 << 20              # > the 126 MB L2
# algorithmic FLOPs credited to each kernel, in units of T*h*m*dh
KERNEL_FLOPS = {"gdpa_fwd_sm100": 4, "gdpa_bwd_sm100": 8, "gdpa_simt_fwd": 4,
                "gdpa_simt_bwd_dq": 4, "gdpa_simt_bwd_dkdv": 4}
WG_KERNEL = "gdpa_weight_gen"
TENSOR_KERNELS = {"gdpa_fwd_sm100", "gdpa_bwd_sm100"}
FWD_KERNELS = {"gdpa_fwd_sm100", "gdpa_simt_fwd"}
# Source files whose contents decide each fused kernel's DRAM traffic.
KERNEL_SOURCES = {"gdpa_fwd_sm100": ("fwd_sm100.cu", "sm100.cuh", "gdpa_internal.cuh"),
                  "gdpa_bwd_sm100": ("bwd_sm100.cu", "sm100.cuh", "gdpa_internal.cuh")}
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per unit T*h*m*dh of
# a fused kernel, from one ncu capture: {kernel: {workload id: (bytes per unit,
# sha16 of the kernel's sources at capture time)}}.  An entry whose hash no
# longer matches the sources is not used (the traffic is then reported null).
TRAFFIC_PER_UNIT = {
    # 64-sample cases: workload 5, 582.2 MB read + 36.3 MB written in one launch;
    # workload 4, 347.3 MB + 60.0 MB
    "gdpa_fwd_sm100": {5: (0.0141478, "209e3f60a671ea6a"), 4: (0.0101234, "209e3f60a671ea6a")},
    # workload 5: 734.8 MB read + 581.8 MB written; workload 4: 599.3 MB + 380.3 MB
    "gdpa_bwd_sm100": {5: (0.0301167, "2fe31e59c24fa0ae"), 4: (0.0243502, "2fe31e59c24fa0ae")},
}
# fp32 FFMA peak for the SIMT kernels: 148 SMs * 128 FMA/clk * 2 flop * 1.965 GHz
SIMT_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
# dense bf16 tcgen05 rate of one SM (flop per clock), for the clock-scaled nominal peak
MMA_FLOP_PER_CLK_SM = 8192
# oracle sample per reference step / per cpu_baseline pass: this many fp64 FLOPs
ORACLE_STEP_FLOPS = 6.0e10


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--e2e-chunks", type=int, default=E2E_CHUNKS,
                    help="sample groups of the end-to-end step (copy-in, compute and copy-out "
                         "of successive groups overlap)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-passes", type=int, default=3,
                    help="passes of the oracle over its fixed sample for cpu_baseline")
    ap.add_argument("--samples", type=int, default=0,
                    help="run only the first N samples of the workload (small profiling case)")
    ap.add_argument("--weight-gen", action="store_true",
                    help="linear-map workload only: generate K and V from the context vectors "
                         "(Weight Generation) inside every step, before the GDPA forward")
    ap.add_argument("--bias", action="store_true",
                    help="the biased PFFN variant: key bias b1 [B,h,m] and output bias b2 "
                         "[B,h,dh] (fp32, N(0,1)/2) in every forward and backward")
    ap.add_argument("--pool", type=int, default=0, metavar="S",
                    help="seed-query attention pooling instead of GDPA: S seeds per head attend "
                         "over the workload's jagged tokens (keys and values [T,h,dh])")
    ap.add_argument("--window", type=int, default=0, metavar="W",
                    help="causal sliding-window self-attention of width W on the workload's "
                         "jagged tokens instead of GDPA")
    ap.add_argument("--variant-backward", action="store_true",
                    help="with --pool or --window: every step runs the forward and the backward")
    ap.add_argument("--phi", default=None,
                    choices=["identity", "silu", "softmax", "relu", "gelu"],
                    help="the same workload with another activation (the PFFN variants' phi)")
    return ap.parse_args(argv)


def e2e_chunks(offsets, nchunks):
    """Equal groups of consecutive samples for the end-to-end step: a list of
    ((first sample, end sample), (first token row, end token row)), non-empty,
    in order, covering every sample once."""
    nb = len(offsets) - 1
    bounds = [nb * c // nchunks for c in range(nchunks + 1)]
    return [((b0, b1), (offsets[b0], offsets[b1]))
            for b0, b1 in zip(bounds[:-1], bounds[1:]) if b1 > b0]


def workload(args):
    """The benchmarked workload, with its activation replaced when --phi is given."""
    import synthetic as syn
    wl = syn.WORKLOADS[getattr(args, "workload", DEFAULT_WORKLOAD)]
    if args.phi and args.phi != wl.phi_name:
        code = {v_: k_ for k_, v_ in syn.PHI_NAMES.items()}[args.phi]
        wl = dataclasses.replace(wl, phi=code, name=wl.name.replace(wl.phi_name, args.phi))
    return wl


def metric_name(wl):
    return "GDPA fwd+bwd TFLOP/s" if wl.backward else "GDPA fwd TFLOP/s"


def step_flop_units(wl):
    """Algorithmic FLOPs of one step in units of T*h*m*dh."""
    return FLOPS_FWD + (FLOPS_BWD if wl.backward else 0)


def fwd_bytes(wl, T):
    """Algorithmic HBM bytes of one forward: Q, K, V read once, O written, LSE."""
    e = 2 if wl.dtype.itemsize == 2 else 4
    b = e * (2 * T * wl.h * wl.dh + 2 * wl.B * wl.h * wl.m * wl.dh)
    return b + (4 * T * wl.h if wl.phi_name == "softmax" else 0)


def config_dict(wl, T, n_gpus, subset=None, weight_gen=False, bias=False):
    """The `config` object of the JSON line (identical in both arms)."""
    return {"weight_gen": weight_gen, "bias": bias,
            "workload": wl.name if subset is None else
            f"{wl.name} (first {len(subset)} samples only: profiling case)",
            "B": wl.B if subset is None else len(subset), "h": wl.h, "dh": wl.dh, "m": wl.m,
            "phi": wl.phi_name, "scale": wl.scale, "lengths": wl.lengths,
            "backward": wl.backward, "tokens_per_rank": int(T),
            "parallelism": f"replicas x{n_gpus} (samples independent)",
            "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MB write outside the "
                  "per-step events)"}


def sources_sha16(kernel):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, ()):
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(kernel, wid, units):
    """DRAM bytes of one launch from the recorded capture, or None when no
    capture exists for this kernel and workload or its sources changed since."""
    ent = TRAFFIC_PER_UNIT.get(kernel, {}).get(wid)
    if not ent or ent[1] != sources_sha16(kernel):
        return None
    return ent[0] * units


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        out = dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                   bf16_sustained=float(d.get("bf16_tflops_sustained") or d["bf16_tflops"]),
                   source="measured", sustained_mhz=None)
        cl = d.get("clocks_under_load") or d.get("sustained_clocks") or {}
        if isinstance(cl, dict):
            for k_ in ("sm_mhz_median", "sm_mhz", "median_sm_mhz"):
                if isinstance(cl.get(k_), (int, float)):
                    out["sustained_mhz"] = float(cl[k_])
                    break
        return out
    except (OSError, KeyError, ValueError, TypeError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback",
                    sustained_mhz=1300.0)


def choose_bf16_peak(pk, clk):
    """Burst or sustained dense bf16 peak, from the SM clock this run saw.

    The sustained figure was taken over a seconds-long GEMM loop that settled
    at a lower clock under the power cap; the burst figure applies while the
    clocks stay near their maximum.  The run's median SM clock decides."""
    med = clk.get("sm_mhz") if clk else None
    mx = clk.get("sm_max_mhz") if clk else None
    if med and pk.get("sustained_mhz") and med <= 1.05 * pk["sustained_mhz"]:
        return pk["bf16_sustained"], (f"{pk['source']} bf16 dense, sustained: median SM clock "
                                      f"{med:.0f} MHz is at the sustained run's "
                                      f"{pk['sustained_mhz']:.0f} MHz")
    why = (f"median SM clock {med:.0f} of {mx:.0f} MHz" if med and mx else "no clock record")
    return pk["bf16"], f"{pk['source']} bf16 dense, burst ({why})"


# --------------------------------------------------------------------------
# CPU oracle (the reported baseline; the oracle as it stands)


def _oracle_unit_flops(n, wl):
    return step_flop_units(wl) * int(n) * wl.h * wl.m * wl.dh


def oracle_sample(wl, lengths, budget=ORACLE_STEP_FLOPS):
    """A fixed seeded choice of samples whose oracle FLOPs fill `budget`
    (the same choice in the cpu_baseline leg and the reference arm)."""
    import numpy as np
    order = np.random.default_rng(1234).permutation(len(lengths))
    pick, acc = [], 0
    for b in order:
        f = _oracle_unit_flops(lengths[b], wl)
        if pick and acc + f > budget:
            continue
        pick.append(int(b))
        acc += f
        if acc >= 0.9 * budget:
            break
    return sorted(pick)


def run_oracle_sample(wl, inputs):
    import oracle
    d = inputs
    t = time.perf_counter()
    oracle.fwd(d["q"], d["k"], d["v"], d["offsets"], wl.phi_name, wl.scale)
    if wl.backward:
        oracle.bwd(d["q"], d["k"], d["v"], d["dout"], d["offsets"], wl.phi_name, wl.scale)
    dt = time.perf_counter() - t
    flops = sum(_oracle_unit_flops(n, wl) for n in d["lengths"])
    return flops, dt, int(d["lengths"].sum())


def oracle_inputs(wl, samples):
    """Host inputs of the chosen samples (the activation does not change them)."""
    import synthetic as syn
    return syn.make_inputs(wl.wid, samples=samples, backward=wl.backward)


def oracle_desc(wl, samples, tokens):
    return (f"{len(samples)} of {wl.B} samples ({tokens} tokens, all {wl.h} heads), "
            f"{'fwd+bwd' if wl.backward else 'fwd'}, fixed seeded choice of "
            f"~{ORACLE_STEP_FLOPS / 1e9:.0f} GFLOP")


# --------------------------------------------------------------------------
# clocks during the timed region


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                cols = [c.strip() for c in line.split(",")]
                if len(cols) < 9:
                    continue
                try:
                    sm.append(float(cols[1]))
                    mx = float(cols[2])
                except ValueError:
                    continue
                for nm, c in zip(names, cols[5:9]):
                    if c.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------


def emit(obj):
    print(json.dumps(obj), flush=True)


def aggregate(ms, flops, tokens, launches, world, dist=None, device=None):
    """Whole-job numbers from per-rank ones: the max of the per-rank device
    times, the sums of FLOPs, tokens and kernel launches.  Every rank takes
    the same two collectives in the same order."""
    if world > 1:
        import torch
        t = torch.tensor([ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        u = torch.tensor([flops, tokens, launches], dtype=torch.float64, device=device)
        dist.all_reduce(u, op=dist.ReduceOp.SUM)
        ms, (flops, tokens, launches) = t.item(), u.tolist()
    return {"ms_max": ms, "flops": flops, "tokens": tokens, "launches": int(launches),
            "tflops": flops / (ms / 1e3) / 1e12 if ms > 0 else 0.0,
            "tokens_per_s": tokens / (ms / 1e3) if ms > 0 else 0.0}


def torchrun_command(args_list, n, port):
    """The torchrun command line that runs this script on n local ranks."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={port}",
            os.path.abspath(__file__), *args_list]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def world_from_env(args):
    """(rank, world, local_rank); raises when a torchrun world disagrees with --gpus."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if "WORLD_SIZE" in os.environ and world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}")
    return rank, world, local_rank


def run_reference(args, rank):
    """The oracle, as it stands, on the host cores; rank 0 only."""
    if rank != 0:
        return
    import synthetic as syn
    wl = workload(args)
    lengths = syn.lengths(wl)
    samples = oracle_sample(wl, lengths)
    inputs = oracle_inputs(wl, samples)
    import oracle
    threads = oracle.max_threads()
    for _ in range(args.warmup):
        run_oracle_sample(wl, inputs)
    flops = secs = 0.0
    tokens = 0
    for _ in range(args.steps):
        f, dt, tk = run_oracle_sample(wl, inputs)
        flops += f
        secs += dt
        tokens += tk
    value = flops / secs / 1e12
    emit({"impl": "reference", "metric": metric_name(wl), "value": value,
          "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
          "ms_per_step": 1e3 * secs / max(args.steps, 1), "higher_is_better": True,
          "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
          "config": config_dict(wl, int(lengths.sum()), args.gpus,
                                weight_gen=bool(getattr(args, "weight_gen", False))),
          "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                           "sample": oracle_desc(wl, samples, tokens // max(args.steps, 1))},
          "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                  "d2h_bytes_per_step": 0},
          "tokens_per_s": tokens / secs})


def variant_flops(kind, lengths, h, dh, S=0, window=0):
    """Algorithmic FLOPs of one forward of an attention variant over a jagged
    batch: pooling 4*S*T*h*dh (S seeds x n_b keys per sample); the causal
    window 4*h*dh * sum over tokens of the keys in their window, where a
    sample of n tokens holds n(n+1)/2 (n <= W) or W*n - W(W-1)/2 of them."""
    n = [int(x) for x in lengths]
    if kind == "pool":
        return 4.0 * S * sum(n) * h * dh
    W = int(window)
    keys = sum(x * (x + 1) // 2 if x <= W else W * x - W * (W - 1) // 2 for x in n)
    return 4.0 * h * dh * keys


VARIANT_KERNELS = {"pool": ("gdpa_pool_fwd_sm100", "gdpa_pool_bwd_sm100"),
                   "window": ("gdpa_window_fwd_sm100", "gdpa_window_bwd_sm100")}


def variant_oracle_sample(lengths, flops_of, budget=ORACLE_STEP_FLOPS):
    """A fixed seeded choice of samples whose oracle FLOPs fill `budget`."""
    import numpy as np
    order = np.random.default_rng(1234).permutation(len(lengths))
    pick, acc = [], 0.0
    for b in order:
        f = flops_of([lengths[b]])
        if pick and acc + f > budget:
            break
        pick.append(int(b))
        acc += f
    return sorted(pick)


def run_variant(args, rank, world, local_rank):
    """Seed-query pooling (--pool S) or the causal sliding window (--window W)
    over the jagged tokens of a workload: per-step device events with the L2
    flushed between steps, max over ranks, the kernel's roofline, the oracle
    on a bounded sample, and an end-to-end pass from pinned host memory."""
    import numpy as np
    import torch
    import torch.distributed as dist

    from recsys_context_personalised_b200 import gdpa as G
    import synthetic as syn

    kind = "pool" if args.pool else "window"
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    wl = syn.WORKLOADS[args.workload]
    lens = syn.lengths(wl, seed=rank)
    if 0 < args.samples < len(lens):
        lens = lens[:args.samples]          # the small profiling case
    offs = syn.offsets_from_lengths(lens)
    B, T, h, dh = len(lens), int(offs[-1]), wl.h, wl.dh
    S, W = int(args.pool), int(args.window)
    scale = 1.0 / dh ** 0.5
    gen = torch.Generator(device=dev)

    def draw(tid, *shape):
        gen.manual_seed(1_000_003 * (rank + 1) + tid)
        return torch.randn(*shape, generator=gen, device=dev).to(torch.bfloat16)

    k, v = draw(1, T, h, dh), draw(2, T, h, dh)
    q = draw(0, h, S, dh) if kind == "pool" else draw(0, T, h, dh)
    bwd = bool(args.variant_backward)
    off = torch.tensor(offs, dtype=torch.int32, device=dev)
    shape = (B, T, int(lens.max()))
    if kind == "pool":
        o = torch.empty((B, h, S, dh), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, h, S), dtype=torch.float32, device=dev)
        n_ws = ctypes_size(G.load().gdpa_pool_workspace_size, B, h, dh, S)
    else:
        o = torch.empty_like(q)
        lse = torch.empty((h, T), dtype=torch.float32, device=dev)
        n_ws = ctypes_size(G.load().gdpa_window_workspace_size, B, h, dh, T)
    ws = torch.empty(max(n_ws, 1), dtype=torch.uint8, device=dev)
    if bwd:
        dout = draw(3, *o.shape)
        dk, dv = torch.empty_like(k), torch.empty_like(v)
        dq = (torch.empty((h, S, dh), dtype=torch.float32, device=dev) if kind == "pool"
              else torch.empty_like(q))
        n_wb = (ctypes_size(G.load().gdpa_pool_bwd_workspace_size, B, h, dh, S, T)
                if kind == "pool" else
                ctypes_size(G.load().gdpa_window_bwd_workspace_size, B, h, dh, T))
        ws_b = torch.empty(max(n_wb, 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    launches = [0]

    def step(q_=q, k_=k, v_=v, o_=o):
        if kind == "pool":
            G.pool_fwd(q_, off, k_, v_, scale, None, o=o_, lse=lse, ws=ws, stream=stream,
                       shape=shape)
        else:
            G.window_fwd(q_, off, k_, v_, W, scale, None, o=o_, lse=lse, ws=ws, stream=stream,
                         shape=shape)
        launches[0] += G.last_launch_count()
        if bwd and kind == "pool":
            G.pool_bwd(q_, off, k_, v_, o_, lse, dout, scale, None, dk=dk, dv=dv, dseeds=dq,
                       ws=ws_b, stream=stream, shape=shape)
            launches[0] += G.last_launch_count()
        elif bwd:
            G.window_bwd(q_, off, k_, v_, o_, lse, dout, W, scale, None, dq=dq, dk=dk, dv=dv,
                         ws=ws_b, stream=stream, shape=shape)
            launches[0] += G.last_launch_count()

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    if G.workspace_status(ws):
        raise RuntimeError("device-side status error during warm-up")

    clocks = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    G.timing_enable(True)
    launches[0] = 0
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    per_kernel = G.timing_read()
    G.timing_enable(False)
    clk = clocks.stop()
    if G.workspace_status(ws) or (bwd and G.workspace_status(ws_b)):
        raise RuntimeError("device-side status error in the timed steps")
    ms = sum(e0.elapsed_time(e1) for e0, e1 in evs)
    fwd_flops = variant_flops(kind, lens, h, dh, S, W)
    flops = fwd_flops * (3.0 if bwd else 1.0)      # the backward credits 8 per 4 of the forward
    agg = aggregate(ms, flops * args.steps, float(T) * args.steps, float(launches[0]), world,
                    dist, dev)
    pk = peaks()
    bf16_peak, peak_why = choose_bf16_peak(pk, clk)
    names = VARIANT_KERNELS[kind] if bwd else VARIANT_KERNELS[kind][:1]
    name = max(names, key=lambda k_: per_kernel.get(k_, (0, 0.0))[1])
    nl, tot_ms = per_kernel.get(name, (0, 0.0))
    avg_ms = tot_ms / max(nl, 1)
    kflops = fwd_flops * (2.0 if name.endswith("bwd_sm100") else 1.0)
    ach = kflops / (avg_ms / 1e3) / 1e12 if avg_ms > 0 else 0.0
    roof = {"bound": "tensor", "achieved": ach, "peak": bf16_peak, "unit": "TFLOP/s",
            "frac": ach / bf16_peak, "peak_source": peak_why, "kernel": name, "traffic": None,
            "traffic_source": "null: no capture of this kernel", "launches": nl,
            "avg_ms": avg_ms}
    kernels = {k_: {"launches": v_[0], "ms": v_[1], "share": v_[1] / max(ms, 1e-9)}
               for k_, v_ in per_kernel.items()}

    # end to end: pinned host inputs in, the call, O out, every step (one stream)
    e2e = None
    if not args.no_e2e and args.e2e_steps > 0:
        ins = ([k, v] if kind == "pool" else [q, k, v]) + ([dout] if bwd else [])
        outs = [o] + ([dq, dk, dv] if bwd else [])
        h_in = [x.cpu().pin_memory() for x in ins]
        h_off = torch.tensor(offs, dtype=torch.int32).pin_memory()
        h_out = [torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in outs]
        h2d = sum(x.numel() * x.element_size() for x in h_in) + h_off.numel() * 4
        d2h = sum(x.numel() * x.element_size() for x in h_out)

        def e2e_step():
            off.copy_(h_off, non_blocking=True)
            for dst, src in zip(ins, h_in):
                dst.copy_(src, non_blocking=True)
            step()
            for dst, src in zip(h_out, outs):
                dst.copy_(src, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        ea = aggregate(e0.elapsed_time(e1), flops * args.e2e_steps, 0.0, 0.0, world, dist, dev)
        e2e = {"value": ea["tflops"], "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "steps": args.e2e_steps,
               "ms_per_step": ea["ms_max"] / args.e2e_steps,
               "api": f"recsys_context_personalised_b200.gdpa.{kind}_fwd"
                      f"{f' + {kind}_bwd' if bwd else ''} with inputs copied from and outputs "
                      "copied to pinned host memory every step (one stream)"}
        del h_in, h_out

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        mult = 3.0 if bwd else 1.0
        pick = variant_oracle_sample(lens, lambda n_: mult * variant_flops(kind, n_, h, dh, S, W))
        rows = np.concatenate([np.arange(offs[b], offs[b + 1]) for b in pick]).astype(np.int64)
        sub_off = syn.offsets_from_lengths([lens[b] for b in pick])
        ridx = torch.tensor(rows, device=dev)
        kh, vh = (x.index_select(0, ridx).float().cpu().numpy() for x in (k, v))
        qh = (q.float().cpu().numpy() if kind == "pool" else
              q.index_select(0, ridx).float().cpu().numpy())
        gh = None
        if bwd:
            gh = (dout.index_select(0, torch.tensor(pick, device=dev)) if kind == "pool" else
                  dout.index_select(0, ridx)).float().cpu().numpy()
        f = dt = 0.0
        for _ in range(max(args.cpu_passes, 1)):
            t0 = time.perf_counter()
            if kind == "pool":
                oracle.pool_fwd(qh, kh, vh, sub_off, scale)
                if bwd:
                    oracle.pool_bwd(qh, kh, vh, gh, sub_off, scale)
            else:
                oracle.win_fwd(qh, kh, vh, sub_off, W, scale)
                if bwd:
                    oracle.win_bwd(qh, kh, vh, gh, sub_off, W, scale)
            dt += time.perf_counter() - t0
            f += mult * variant_flops(kind, [lens[b] for b in pick], h, dh, S, W)
        cpu = {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.max_threads(),
               "kind": "oracle",
               "sample": f"{len(pick)} of {B} samples ({len(rows)} tokens, all {h} heads), "
                         f"{'fwd+bwd' if bwd else 'fwd'}, fixed seeded choice, "
                         f"{args.cpu_passes} passes, {dt:.1f} s"}

    if rank == 0:
        what = (f"hsp_seed_pool_S{S}" if kind == "pool" else f"sliding_window_W{W}")
        emit({"metric": ("HSP seed-query pooling " if kind == "pool" else
                         "sliding-window self-attention ") + ("fwd+bwd" if bwd else "fwd") +
                        " TFLOP/s",
              "value": agg["tflops"], "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
              "warmup": args.warmup, "ms_per_step": agg["ms_max"] / args.steps,
              "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
              "data": "synthetic",
              "config": {"workload": f"{what}_tokens_of_{wl.name}" +
                                     (f" (first {B} samples only: profiling case)"
                                      if B < wl.B else ""), "B": B, "h": h, "dh": dh,
                         "seeds": S or None, "window": W or None, "lengths": wl.lengths,
                         "tokens_per_rank": T, "scale": scale,
                         "inputs": "N(0,1) bf16 from a seeded torch generator per tensor",
                         "parallelism": f"replicas x{world} (samples independent)",
                         "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MB write "
                               "outside the per-step events)"},
              "pct_of_bf16_peak": 100.0 * agg["tflops"] / (world * bf16_peak),
              "flops_per_step": flops, "backward": bwd, "tokens_per_s": agg["tokens_per_s"],
              "gpu_launches": agg["launches"], "kernels": kernels, "roofline": roof,
              "cpu_baseline": cpu, "e2e": e2e, "clocks": clk})
    if world > 1:
        dist.destroy_process_group()


def ctypes_size(fn, *args_):
    """Call a `*_workspace_size` entry point; the size in bytes."""
    import ctypes
    n = ctypes.c_size_t()
    rc = fn(*args_, ctypes.byref(n))
    if rc:
        raise RuntimeError(f"workspace size query failed with code {rc}")
    return int(n.value)


def main(argv=None):
    args = parse(argv)
    if args.pool and args.window:
        raise SystemExit("bench.py: --pool and --window are separate workloads")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        argv = sys.argv[1:] if argv is None else list(argv)
        cmd = torchrun_command(argv, args.gpus, _free_port())
        raise SystemExit(subprocess.call(cmd))
    rank, world, local_rank = world_from_env(args)
    if args.impl == "reference":
        if args.pool or args.window:
            raise SystemExit("bench.py: the reference arm times the GDPA workloads; the "
                             "attention variants report the oracle as cpu_baseline")
        run_reference(args, rank)
        return
    if args.pool or args.window:
        run_variant(args, rank, world, local_rank)
        return

    import torch
    import torch.distributed as dist

    import recsys_context_personalised_b200 as pkg
    from recsys_context_personalised_b200 import gdpa as G
    import synthetic as syn

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    wl = workload(args)
    subset = list(range(args.samples)) if 0 < args.samples < wl.B else None
    d = syn.make_inputs(wl.wid, device=dev, seed=rank, backward=wl.backward, samples=subset)
    q, k, v, g = d["q"], d["k"], d["v"], d.get("dout")
    T = int(d["offsets"][-1])
    off = torch.tensor(d["offsets"], dtype=torch.int32, device=dev)
    p = pkg.problem_for(q, k, d["offsets"], wl.phi_name, wl.scale,
                        max_n=int(d["lengths"].max()))
    o = torch.empty_like(q)
    lse = torch.empty((wl.h, T), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)) \
        if wl.backward else (None, None, None)
    ws_f = pkg.workspace(pkg.fwd_workspace_bytes(p), dev)
    ws_b = pkg.workspace(pkg.bwd_workspace_bytes(p), dev) if wl.backward else None
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    launches = [0]

    wg = None
    if args.weight_gen:
        if wl.kv_recipe != "linear_map" or subset is not None:
            raise SystemExit("bench.py: --weight-gen needs the linear-map workload (2), all samples")
        wg = {x: syn.weight_gen_factors(wl.wid, x, seed=rank, device=dev) for x in ("k", "v")}

    b1 = b2 = db1 = db2 = None
    if args.bias:            # the biased PFFN variant: phi(s Q K^T + b1) V + b2
        bgen = torch.Generator(device=dev)
        bgen.manual_seed(7919 + rank)
        b1 = 0.5 * torch.randn((k.shape[0], wl.h, wl.m), generator=bgen, device=dev)
        b2 = 0.5 * torch.randn((k.shape[0], wl.h, wl.dh), generator=bgen, device=dev)
        db1, db2 = torch.empty_like(b1), torch.empty_like(b2)

    def step():
        if wg is not None:       # K, V = reshape(W c_b) for every sample, then the GDPA forward
            G.weight_gen(wg["k"][0], wg["k"][1], y=k.view(wl.B, -1), stream=stream)
            launches[0] += 1
            G.weight_gen(wg["v"][0], wg["v"][1], y=v.view(wl.B, -1), stream=stream)
            launches[0] += 1
        if args.bias:
            G.fwd_bias(p, q, off, k, v, b1, b2, o=o, lse=lse, ws=ws_f, stream=stream)
        else:
            G.fwd(p, q, off, k, v, o=o, lse=lse, ws=ws_f, stream=stream)
        launches[0] += G.last_launch_count()
        if wl.backward:
            if args.bias:
                G.bwd_bias(p, q, off, k, v, b1, b2, o, lse, g, dq=dq, dk=dk, dv=dv, db1=db1,
                           db2=db2, ws=ws_b, stream=stream)
            else:
                G.bwd(p, q, off, k, v, o, lse, g, dq=dq, dk=dk, dv=dv, ws=ws_b, stream=stream)
            launches[0] += G.last_launch_count()

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    if pkg.workspace_status(ws_f) or (ws_b is not None and pkg.workspace_status(ws_b)):
        raise RuntimeError("device-side status error during warm-up")

    # ---- timed region: per-step device events, L2 flushed between steps ----
    clocks = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    G.timing_enable(True)
    launches[0] = 0
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    per_kernel = G.timing_read()
    G.timing_enable(False)
    clk = clocks.stop()
    ms = sum(e0.elapsed_time(e1) for e0, e1 in evs)
    unit_flops = float(T) * wl.h * wl.m * wl.dh
    agg = aggregate(ms, step_flop_units(wl) * unit_flops * args.steps, float(T) * args.steps,
                    float(launches[0]), world, dist, dev)
    ms_max, value, n_launch = agg["ms_max"], agg["tflops"], agg["launches"]

    # ---- rooflines: dominant kernel, and the forward kernel on its own ----
    pk = peaks()
    bf16_peak, peak_why = choose_bf16_peak(pk, clk)
    fp32 = wl.dtype == torch.float32
    nominal = None
    if clk and clk.get("sm_mhz"):
        nominal = 148 * MMA_FLOP_PER_CLK_SM * clk["sm_mhz"] * 1e6 / 1e12

    def roofline(name):
        nl, tot_ms = per_kernel[name]
        avg_ms = tot_ms / max(nl, 1)
        flops = KERNEL_FLOPS.get(name, 0) * unit_flops
        tflops = flops / (avg_ms / 1e3) / 1e12
        if name in FWD_KERNELS and not fp32 and wl.wid == 2:
            # m = 256: below the ridge (171 flop/B); judged on HBM bytes
            nbytes = fwd_bytes(wl, T)
            gbs = nbytes / (avg_ms / 1e3) / 1e9
            r = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s",
                 "frac": gbs / pk["hbm"], "peak_source": f"{pk['source']} HBM copy",
                 "algorithmic_bytes": nbytes, "tflops": tflops,
                 "frac_of_bf16_peak": tflops / bf16_peak}
        elif name in TENSOR_KERNELS:
            r = {"bound": "tensor", "achieved": tflops, "peak": bf16_peak, "unit": "TFLOP/s",
                 "frac": tflops / bf16_peak, "peak_source": peak_why,
                 "frac_of_sustained": tflops / pk["bf16_sustained"],
                 "frac_of_nominal_at_clock": tflops / nominal if nominal else None}
        else:
            r = {"bound": "alu", "achieved": tflops, "peak": SIMT_PEAK_TFLOPS, "unit": "TFLOP/s",
                 "frac": tflops / SIMT_PEAK_TFLOPS,
                 "peak_source": "fp32 FFMA: 148 SMs x 128 lanes x 2 flop x 1.965 GHz"}
        t_ = traffic_for(name, wl.wid, unit_flops) if subset is None else None
        r.update(kernel=name, traffic=t_, launches=nl, avg_ms=avg_ms,
                 traffic_source=("ncu DRAM bytes per T*h*m*dh of a capture of this kernel "
                                 "source, scaled to the launch" if t_ else
                                 "null: no capture of the current kernel source"))
        return r

    credited = [k_ for k_ in per_kernel if KERNEL_FLOPS.get(k_, 0)]
    top = max(credited or per_kernel, key=lambda k_: per_kernel[k_][1])
    roof = roofline(top)
    fwd_name = next((k_ for k_ in per_kernel if k_ in FWD_KERNELS), None)
    roof_fwd = roofline(fwd_name) if fwd_name else None
    roof_wg = None
    if wg is not None and WG_KERNEL in per_kernel:
        # HBM-bound map: w (fp32) and ctx read, y (bf16) written, per launch
        nl, tot_ms = per_kernel[WG_KERNEL]
        avg = tot_ms / max(nl, 1)
        F = wl.h * wl.m * wl.dh
        nbytes = F * syn.CTX_DIM * 4 + wl.B * syn.CTX_DIM * 4 + wl.B * F * 2
        gbs = nbytes / (avg / 1e3) / 1e9
        roof_wg = {"bound": "hbm", "kernel": WG_KERNEL, "achieved": gbs, "peak": pk["hbm"],
                   "unit": "GB/s", "frac": gbs / pk["hbm"], "algorithmic_bytes": nbytes,
                   "launches": nl, "avg_ms": avg, "peak_source": f"{pk['source']} HBM copy",
                   "tflops": 2.0 * wl.B * F * syn.CTX_DIM / (avg / 1e3) / 1e12}
    kernels = {k_: {"launches": v_[0], "ms": v_[1], "share": v_[1] / max(ms, 1e-9)}
               for k_, v_ in per_kernel.items()}

    # ---- end to end through host buffers ----
    # The step again, through the public API, from pinned host memory: the
    # batch is cut into E2E_CHUNKS equal groups of samples, each its own
    # fwd (+ bwd) call on views of the device tensors.  One stream copies chunk
    # inputs in, one computes, one copies chunk outputs back, so the two PCIe
    # directions and the compute overlap; per-chunk events order every reuse
    # of a buffer (also from one step to the next).
    e2e = None
    if not args.no_e2e and args.e2e_steps > 0 and not args.bias:
        o_full = o.clone()          # O of the full-batch call (the forward is deterministic)
        ins = [q, k, v] + ([g] if wl.backward else [])
        outs = [o] + ([dq, dk, dv] if wl.backward else [])
        h_in = [x.cpu().pin_memory() for x in ins]
        h_out = [torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in outs]
        token_major_in = [True, False, False, True]
        token_major_out = [True, True, False, False]
        offs = [int(x) for x in d["offsets"]]
        chunks = []
        for (b0, b1), (t0_, t1_) in e2e_chunks(offs, max(1, args.e2e_chunks)):
            coff = [x - t0_ for x in offs[b0:b1 + 1]]
            cp_ = pkg.problem_for(q[t0_:t1_], k[b0:b1], coff, wl.phi_name, wl.scale,
                                  max_n=max(coff[i + 1] - coff[i] for i in range(b1 - b0)))
            chunks.append(dict(
                rows=(t0_, t1_), smp=(b0, b1), p=cp_,
                hoff=torch.tensor(coff, dtype=torch.int32).pin_memory(),
                off=torch.empty(len(coff), dtype=torch.int32, device=dev),
                lse=torch.empty((wl.h, max(t1_ - t0_, 1)), dtype=torch.float32, device=dev),
                wsf=pkg.workspace(pkg.fwd_workspace_bytes(cp_), dev),
                wsb=pkg.workspace(pkg.bwd_workspace_bytes(cp_), dev) if wl.backward else None,
                loaded=torch.cuda.Event(), computed=torch.cuda.Event(), sent=torch.cuda.Event()))
        h2d = sum(x.numel() * x.element_size() for x in h_in) + \
            sum(c_["hoff"].numel() * 4 for c_ in chunks)
        d2h = sum(x.numel() * x.element_size() for x in h_out)
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        first = [True]

        def rng(c_, tok):
            (t0_, t1_), (b0, b1) = c_["rows"], c_["smp"]
            return slice(t0_, t1_) if tok else slice(b0, b1)

        def e2e_step():
            for c_ in chunks:
                with torch.cuda.stream(s_in):
                    if not first[0]:
                        s_in.wait_event(c_["computed"])       # last step's compute read them
                    c_["off"].copy_(c_["hoff"], non_blocking=True)
                    for dst, src, tok in zip(ins, h_in, token_major_in):
                        dst[rng(c_, tok)].copy_(src[rng(c_, tok)], non_blocking=True)
                    c_["loaded"].record(s_in)
            for c_ in chunks:
                stream.wait_event(c_["loaded"])
                if not first[0]:
                    stream.wait_event(c_["sent"])             # last step's outputs copied out
                tr, sr = rng(c_, True), rng(c_, False)
                cl = c_["lse"][:, :c_["rows"][1] - c_["rows"][0]]
                G.fwd(c_["p"], q[tr], c_["off"], k[sr], v[sr], o=o[tr], lse=cl, ws=c_["wsf"],
                      stream=stream)
                if wl.backward:
                    G.bwd(c_["p"], q[tr], c_["off"], k[sr], v[sr], o[tr], cl, g[tr], dq=dq[tr],
                          dk=dk[sr], dv=dv[sr], ws=c_["wsb"], stream=stream)
                c_["computed"].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(c_["computed"])
                    for dst, src, tok in zip(h_out, outs, token_major_out):
                        dst[rng(c_, tok)].copy_(src[rng(c_, tok)], non_blocking=True)
                    c_["sent"].record(s_out)
            first[0] = False

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        e0.record(s_in)
        for _ in range(args.e2e_steps):
            e2e_step()
        s_out.wait_stream(stream)
        s_out.wait_stream(s_in)
        e1.record(s_out)
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
        barrier()
        bad = [pkg.workspace_status(c_["wsf"]) or
               (wl.backward and pkg.workspace_status(c_["wsb"])) for c_ in chunks]
        if any(bad):
            raise RuntimeError("device-side status error in the end-to-end steps")
        if not torch.equal(h_out[0], o_full.cpu()):
            raise RuntimeError("end-to-end O differs from the full-batch O")
        ea = aggregate(e0.elapsed_time(e1),
                       step_flop_units(wl) * unit_flops * args.e2e_steps, 0.0, 0.0, world, dist,
                       dev)
        ems = ea["ms_max"]
        e2e = {"value": ea["tflops"], "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": args.e2e_steps, "ms_per_step": ems / args.e2e_steps,
               "wall_ms_per_step": 1e3 * wall / args.e2e_steps,
               "api": (f"recsys_context_personalised_b200.gdpa fwd"
                       f"{'/bwd' if wl.backward else ''} on {len(chunks)} sample chunks copied "
                       "from and to pinned host memory; copy-in, compute and copy-out on three "
                       "streams")}
        del h_in, h_out, chunks, o_full

    # ---- CPU oracle baseline (rank 0 at N=1 only) ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        samples = oracle_sample(wl, syn.lengths(wl))
        inputs = oracle_inputs(wl, samples)
        f = dt = 0.0
        tk = 0
        for _ in range(max(args.cpu_passes, 1)):
            f_, dt_, tk = run_oracle_sample(wl, inputs)
            f += f_
            dt += dt_
        cpu = {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.max_threads(),
               "kind": "oracle",
               "sample": oracle_desc(wl, samples, tk) + f", {args.cpu_passes} passes, "
                                                       f"{dt:.1f} s"}

    if rank == 0:
        emit({"metric": metric_name(wl), "value": value, "unit": "TFLOP/s",
              "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
              "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
              "vs_baseline": None, "dtype": "f32" if fp32 else "bf16", "data": "synthetic",
              "config": config_dict(wl, T, world, subset, bool(args.weight_gen),
                                    bool(args.bias)),
              "pct_of_bf16_peak": None if fp32 else 100.0 * value / (world * bf16_peak),
              "bf16_peak": None if fp32 else {"value": bf16_peak, "source": peak_why,
                                              "nominal_at_median_clock": nominal},
              "tokens_per_s": agg["tokens_per_s"],
              "fwd_flops_per_step": FLOPS_FWD * unit_flops,
              "bwd_flops_per_step": FLOPS_BWD * unit_flops if wl.backward else 0.0,
              "gpu_launches": n_launch, "kernels": kernels, "roofline": roof,
              "roofline_fwd": roof_fwd, "roofline_weight_gen": roof_wg, "cpu_baseline": cpu,
              "e2e": e2e, "clocks": clk})
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
