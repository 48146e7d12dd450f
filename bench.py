#!/usr/bin/env python
"""GDPA benchmark: forward + backward TFLOP/s on one B200 (or N replicas).

One step = the whole GDPA hot path over one synthetic batch: tile scheduling,
the fused forward (S = s Q K^T, P = phi(S), O = P V, softmax statistics) and
the fused backward (dQ, dK, dV).  The workload is the largest jagged bf16
softmax problem: B = 1024 samples with power-law (alpha = 1.5) history lengths
on [32, 4096], h = 16 heads, dh = 64, m = 2048 context keys per sample and
head, scale 1/sqrt(dh).

Throughput counts algorithmic FLOPs only: forward 4*T*h*m*dh, backward
8*T*h*m*dh (the recomputation of S in the backward is not credited).

Multi-GPU: samples are independent and the op has no exchange step, so N
ranks run N independent batches (weak scaling, no collective on the data
path; a barrier and one max-reduction of the timings only).

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload (rank 0 only), in the same units.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = 5
E2E_CHUNKS = 8                          # sample groups of the end-to-end step
FLOPS_FWD, FLOPS_BWD = 4, 8            # x T*h*m*dh
# algorithmic FLOPs credited to each kernel, in units of T*h*m*dh
KERNEL_FLOPS = {"gdpa_fwd_sm100": 4, "gdpa_bwd_sm100": 8, "gdpa_simt_fwd": 4,
                "gdpa_simt_bwd_dq": 4, "gdpa_simt_bwd_dkdv": 4}
TENSOR_KERNELS = {"gdpa_fwd_sm100", "gdpa_bwd_sm100"}
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per unit T*h*m*dh of
# the fused kernels, from one ncu capture on the first 64 samples of this
# workload (T = 20,846; `bench.py --samples 64 --steps 1 --warmup 1`):
# backward 743,162,880 + 589,410,048 B, forward 580,738,816 + 34,836,480 B.
# A launch's traffic is this times its units; valid only for the kernels as
# captured (set an entry to None when its kernel changes).
_CAPTURE_UNITS = 20846 * 16 * 2048 * 64
TRAFFIC_PER_UNIT = {"gdpa_bwd_sm100": (743162880 + 589410048) / _CAPTURE_UNITS,
                    "gdpa_fwd_sm100": (580738816 + 34836480) / _CAPTURE_UNITS}
# fp32 FFMA peak for the SIMT kernels: 148 SMs * 128 FMA/clk * 2 flop * 1.965 GHz
SIMT_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--samples", type=int, default=0,
                    help="run only the first N samples of the workload (small profiling case)")
    ap.add_argument("--phi", default=None,
                    choices=["identity", "silu", "softmax", "relu", "gelu"],
                    help="the same workload with another activation (the PFFN variants' phi)")
    return ap.parse_args()


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
    wl = syn.WORKLOADS[WORKLOAD]
    if args.phi and args.phi != wl.phi_name:
        code = {v_: k_ for k_, v_ in syn.PHI_NAMES.items()}[args.phi]
        wl = dataclasses.replace(wl, phi=code, name=wl.name.replace(wl.phi_name, args.phi))
    return wl


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sustained=d["bf16_tflops_sustained"], source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# --------------------------------------------------------------------------
# CPU oracle timing (the reported baseline; the oracle as it stands)


def _oracle_unit_flops(n, wl):
    return (FLOPS_FWD + FLOPS_BWD) * int(n) * wl.h * wl.m * wl.dh


def time_oracle(wl, lengths, seconds, seed=0):
    """Time the oracle's fwd+bwd on a seeded sample of samples (~`seconds`)."""
    import numpy as np

    import oracle
    import synthetic as syn
    rng = np.random.default_rng(1234)
    order = rng.permutation(len(lengths))
    threads = oracle.max_threads()
    # calibrate on one short sample (its h units keep min(h, threads) cores busy)
    probe = [int(next(b for b in order if lengths[b] <= 256))]
    d = syn.make_inputs(wl.wid, samples=probe, backward=True, seed=seed)
    t = time.perf_counter()
    oracle.fwd(d["q"], d["k"], d["v"], d["offsets"], wl.phi_name, wl.scale)
    oracle.bwd(d["q"], d["k"], d["v"], d["dout"], d["offsets"], wl.phi_name, wl.scale)
    dt = max(time.perf_counter() - t, 1e-3)
    per_core = _oracle_unit_flops(lengths[probe[0]], wl) / dt / min(threads, wl.h)
    budget = per_core * threads * seconds
    pick, acc = [], 0
    for b in order:
        f = _oracle_unit_flops(lengths[b], wl)
        if pick and acc + f > budget:
            continue
        pick.append(int(b))
        acc += f
        if acc >= 0.8 * budget:
            break
    return pick, threads


def run_oracle_sample(wl, samples, seed=0):
    import oracle
    import synthetic as syn
    d = syn.make_inputs(wl.wid, samples=samples, backward=True, seed=seed)
    t = time.perf_counter()
    oracle.fwd(d["q"], d["k"], d["v"], d["offsets"], wl.phi_name, wl.scale)
    oracle.bwd(d["q"], d["k"], d["v"], d["dout"], d["offsets"], wl.phi_name, wl.scale)
    dt = time.perf_counter() - t
    flops = sum(_oracle_unit_flops(n, wl) for n in d["lengths"])
    return flops, dt, int(d["lengths"].sum())


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


def run_reference(args, rank):
    """The oracle, as it stands, on the host cores; rank 0 only."""
    if rank != 0:
        return
    import synthetic as syn
    wl = workload(args)
    lengths = syn.lengths(wl)
    total = args.steps + args.warmup
    per_step = max(1.0, min(8.0, 150.0 / max(total, 1)))
    samples, threads = time_oracle(wl, lengths, per_step)
    for _ in range(args.warmup):
        run_oracle_sample(wl, samples)
    flops = secs = 0.0
    tokens = 0
    for _ in range(args.steps):
        f, dt, tk = run_oracle_sample(wl, samples)
        flops += f
        secs += dt
        tokens += tk
    value = flops / secs / 1e12
    sample_desc = (f"{len(samples)} of {wl.B} samples per step ({tokens // max(args.steps, 1)} "
                   f"tokens, all {wl.h} heads), fwd+bwd, seeded choice")
    emit({"impl": "reference", "metric": "GDPA fwd+bwd TFLOP/s", "value": value,
          "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
          "ms_per_step": 1e3 * secs / max(args.steps, 1), "higher_is_better": True,
          "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
          "config": {"workload": wl.name, "B": wl.B, "h": wl.h, "dh": wl.dh, "m": wl.m,
                     "phi": wl.phi_name, "lengths": wl.lengths, "parallelism": "none (CPU)"},
          "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                           "sample": sample_desc},
          "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                  "d2h_bytes_per_step": 0},
          "tokens_per_s": tokens / secs})


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import numpy as np
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
    d = syn.make_inputs(WORKLOAD, device=dev, seed=rank, backward=True, samples=subset)
    q, k, v, g = d["q"], d["k"], d["v"], d["dout"]
    T = int(d["offsets"][-1])
    off = torch.tensor(d["offsets"], dtype=torch.int32, device=dev)
    p = pkg.problem_for(q, k, d["offsets"], wl.phi_name, wl.scale,
                        max_n=int(d["lengths"].max()))
    o = torch.empty_like(q)
    lse = torch.empty((wl.h, T), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_f = pkg.workspace(pkg.fwd_workspace_bytes(p), dev)
    ws_b = pkg.workspace(pkg.bwd_workspace_bytes(p), dev)
    stream = torch.cuda.current_stream()
    launches = [0]

    def step():
        G.fwd(p, q, off, k, v, o=o, lse=lse, ws=ws_f, stream=stream)
        launches[0] += G.last_launch_count()
        G.bwd(p, q, off, k, v, o, lse, g, dq=dq, dk=dk, dv=dv, ws=ws_b, stream=stream)
        launches[0] += G.last_launch_count()

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    if pkg.workspace_status(ws_f) or pkg.workspace_status(ws_b):
        raise RuntimeError("device-side status error during warm-up")

    # ---- timed region (device events; inputs are far larger than L2) ----
    clocks = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    G.timing_enable(True)
    launches[0] = 0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    per_kernel = G.timing_read()
    G.timing_enable(False)
    clk = clocks.stop()
    ms = ev0.elapsed_time(ev1)
    unit_flops = float(T) * wl.h * wl.m * wl.dh
    agg = aggregate(ms, (FLOPS_FWD + FLOPS_BWD) * unit_flops * args.steps, float(T) * args.steps,
                    float(launches[0]), world, dist, dev)
    ms_max, value, n_launch = agg["ms_max"], agg["tflops"], agg["launches"]

    # ---- dominant kernel roofline ----
    pk = peaks()
    credited = {k_: v_ for k_, v_ in per_kernel.items() if KERNEL_FLOPS.get(k_, 0)}
    top = max((credited or per_kernel).items(), key=lambda kv: kv[1][1])
    name, (nl, tot_ms) = top
    avg_ms = tot_ms / max(nl, 1)
    per_launch_flops = KERNEL_FLOPS.get(name, 0) * unit_flops
    achieved = per_launch_flops / (avg_ms / 1e3) / 1e12
    if name in TENSOR_KERNELS:
        roof = {"bound": "tensor", "peak": pk["bf16_sustained"],
                "peak_source": f"{pk['source']} bf16 dense, sustained (kernel timed inside a long step loop)"}
    else:
        roof = {"bound": "alu", "peak": SIMT_PEAK_TFLOPS,
                "peak_source": "fp32 FFMA: 148 SMs x 128 lanes x 2 flop x 1.965 GHz"}
    tpu = TRAFFIC_PER_UNIT.get(name) if WORKLOAD == 5 and wl.phi_name == "softmax" else None
    roof.update(kernel=name, achieved=achieved, unit="TFLOP/s", frac=achieved / roof["peak"],
                traffic=tpu * unit_flops if tpu else None,
                traffic_source=("ncu DRAM bytes of a 64-sample capture, scaled by T*h*m*dh"
                                if tpu else None),
                launches=nl, avg_ms=avg_ms)
    kernels = {k_: {"launches": v_[0], "ms": v_[1], "share": v_[1] / max(ms, 1e-9)}
               for k_, v_ in per_kernel.items()}

    # ---- end to end through host buffers ----
    # The step again, through the public API, from pinned host memory: the
    # batch is cut into E2E_CHUNKS equal groups of samples, each its own
    # fwd + bwd call on views of the device tensors.  One stream copies chunk
    # inputs in, one computes, one copies chunk outputs back, so the two PCIe
    # directions and the compute overlap; per-chunk events order every reuse
    # of a buffer (also from one step to the next).
    e2e = None
    if not args.no_e2e and args.e2e_steps > 0:
        o_full = o.clone()          # O of the full-batch call (the forward is deterministic)
        hq, hk, hv, hg = (x.cpu().pin_memory() for x in (q, k, v, g))
        ho, hdq, hdk, hdv = (torch.empty(x.shape, dtype=x.dtype).pin_memory()
                             for x in (o, dq, dk, dv))
        offs = [int(x) for x in d["offsets"]]
        chunks = []
        for (b0, b1), (t0_, t1_) in e2e_chunks(offs, E2E_CHUNKS):
            coff = [x - t0_ for x in offs[b0:b1 + 1]]
            cp_ = pkg.problem_for(q[t0_:t1_], k[b0:b1], coff, wl.phi_name, wl.scale,
                                  max_n=max(coff[i + 1] - coff[i] for i in range(b1 - b0)))
            chunks.append(dict(
                rows=(t0_, t1_), smp=(b0, b1), p=cp_,
                hoff=torch.tensor(coff, dtype=torch.int32).pin_memory(),
                off=torch.empty(len(coff), dtype=torch.int32, device=dev),
                lse=torch.empty((wl.h, max(t1_ - t0_, 1)), dtype=torch.float32, device=dev),
                wsf=pkg.workspace(pkg.fwd_workspace_bytes(cp_), dev),
                wsb=pkg.workspace(pkg.bwd_workspace_bytes(cp_), dev),
                loaded=torch.cuda.Event(), computed=torch.cuda.Event(), sent=torch.cuda.Event()))
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hg)) + \
            sum(c_["hoff"].numel() * 4 for c_ in chunks)
        d2h = sum(x.numel() * x.element_size() for x in (ho, hdq, hdk, hdv))
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        first = [True]

        def e2e_step():
            for c_ in chunks:
                (t0_, t1_), (b0, b1) = c_["rows"], c_["smp"]
                with torch.cuda.stream(s_in):
                    if not first[0]:
                        s_in.wait_event(c_["computed"])       # last step's compute read them
                    c_["off"].copy_(c_["hoff"], non_blocking=True)
                    for dst, src in ((q, hq), (g, hg)):
                        dst[t0_:t1_].copy_(src[t0_:t1_], non_blocking=True)
                    for dst, src in ((k, hk), (v, hv)):
                        dst[b0:b1].copy_(src[b0:b1], non_blocking=True)
                    c_["loaded"].record(s_in)
            for c_ in chunks:
                (t0_, t1_), (b0, b1) = c_["rows"], c_["smp"]
                stream.wait_event(c_["loaded"])
                if not first[0]:
                    stream.wait_event(c_["sent"])             # last step's outputs copied out
                cq, cg, co, cdq = q[t0_:t1_], g[t0_:t1_], o[t0_:t1_], dq[t0_:t1_]
                ck, cv, cdk, cdv = k[b0:b1], v[b0:b1], dk[b0:b1], dv[b0:b1]
                cl = c_["lse"][:, :t1_ - t0_]
                G.fwd(c_["p"], cq, c_["off"], ck, cv, o=co, lse=cl, ws=c_["wsf"], stream=stream)
                G.bwd(c_["p"], cq, c_["off"], ck, cv, co, cl, cg, dq=cdq, dk=cdk, dv=cdv,
                      ws=c_["wsb"], stream=stream)
                c_["computed"].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(c_["computed"])
                    for dst, src in ((ho, o), (hdq, dq)):
                        dst[t0_:t1_].copy_(src[t0_:t1_], non_blocking=True)
                    for dst, src in ((hdk, dk), (hdv, dv)):
                        dst[b0:b1].copy_(src[b0:b1], non_blocking=True)
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
        bad = [pkg.workspace_status(c_["wsf"]) or pkg.workspace_status(c_["wsb"]) for c_ in chunks]
        if any(bad):
            raise RuntimeError("device-side status error in the end-to-end steps")
        if not torch.equal(ho, o_full.cpu()):
            raise RuntimeError("end-to-end O differs from the full-batch O")
        ea = aggregate(e0.elapsed_time(e1), (FLOPS_FWD + FLOPS_BWD) * unit_flops * args.e2e_steps,
                       0.0, 0.0, world, dist, dev)
        ems = ea["ms_max"]
        e2e = {"value": ea["tflops"], "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": args.e2e_steps, "ms_per_step": ems / args.e2e_steps,
               "wall_ms_per_step": 1e3 * wall / args.e2e_steps,
               "api": (f"recsys_context_personalised_b200.gdpa fwd/bwd on {len(chunks)} sample "
                       "chunks copied from and to pinned host memory; copy-in, compute and "
                       "copy-out on three streams")}
        del hq, hk, hv, hg, ho, hdq, hdk, hdv, chunks, o_full

    # ---- CPU oracle baseline (rank 0 at N=1 only) ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        samples, threads = time_oracle(wl, syn.lengths(wl), args.cpu_seconds)
        f, dt, tk = run_oracle_sample(wl, samples)
        cpu = {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{len(samples)} of {wl.B} samples ({tk} tokens, all {wl.h} heads), "
                         f"fwd+bwd, seeded choice, {dt:.1f} s"}

    if rank == 0:
        emit({"metric": "GDPA fwd+bwd TFLOP/s", "value": value, "unit": "TFLOP/s",
              "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
              "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
              "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
              "config": {"workload": wl.name if subset is None else
                         f"{wl.name} (first {len(subset)} samples only: profiling case)",
                         "B": wl.B if subset is None else len(subset), "h": wl.h, "dh": wl.dh,
                         "m": wl.m, "phi": wl.phi_name, "scale": wl.scale, "lengths": wl.lengths,
                         "tokens_per_rank": T, "parallelism": f"replicas x{world} (samples independent)",
                         "l2": "inputs (K, V 4.3 GB each) far larger than the 126 MB L2; no flush"},
              "pct_of_bf16_peak": 100.0 * value / (world * pk["bf16_sustained"]),
              "tokens_per_s": agg["tokens_per_s"],
              "fwd_flops_per_step": FLOPS_FWD * unit_flops, "bwd_flops_per_step": FLOPS_BWD * unit_flops,
              "gpu_launches": n_launch, "kernels": kernels, "roofline": roof,
              "cpu_baseline": cpu, "e2e": e2e, "clocks": clk})
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
