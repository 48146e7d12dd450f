"""Seeded synthetic inputs for GDPA (Generalized Dot-Product Attention).

This module only draws numbers: it holds none of GDPA's arithmetic. Both the
CPU oracle's tests and the CUDA path's tests and benchmark take their inputs
from here, so that the two sides see the same bits.

Generator.  Every tensor element is a pure function of (seed, workload id,
tensor id, flat element index), so any subset of samples can be regenerated
on its own, on the host or on the device:

* bits(i)   = splitmix64 finaliser of (key + (i + 1) * 0x9E3779B97F4A7C15), the
              counter form of Steele, Lea and Flood's SplitMix64 generator
              ("Fast splittable pseudorandom number generators", OOPSLA 2014);
* uniform   = ((bits >> 11) + 0.5) / 2**53, which lies strictly inside (0, 1);
* normal_i  = Box-Muller on the uniforms of counters 2i and 2i+1 (cosine
              branch only), evaluated in float64, then scaled and rounded once
              to the storage dtype (bf16 round-to-nearest-even, or fp32).

The integer part is exact on every device.  The float64 log/sqrt/cos may
differ by an ulp between host and device libraries, which the single rounding
to bf16/fp32 removes except at exact rounding ties.

Workloads.  The five GDPA workloads are the problem shapes named for this op:
sizes, activations, scales and length distributions (jagged user-history
lengths per sample, one context K/V set per sample and head).  The layout is
token-major jagged Q/O/dO [T, h, dh] with int32 offsets [B+1], and K/V
[B, h, m, dh].
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Iterable, Optional, Sequence

import numpy as np
import torch

PHI_IDENTITY, PHI_SILU, PHI_SOFTMAX = 0, 1, 2
PHI_NAMES = {PHI_IDENTITY: "identity", PHI_SILU: "silu", PHI_SOFTMAX: "softmax", 3: "relu",
             4: "gelu"}

_GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1

# tensor ids inside one workload's counter space
T_LENGTHS, T_Q, T_K, T_V, T_DOUT, T_WK, T_WV, T_CTX = 1, 2, 3, 4, 5, 6, 7, 8


def _to_i64(x: int) -> int:
    """Two's-complement view of a 64-bit unsigned constant, for torch.int64."""
    x &= _MASK64
    return x - (1 << 64) if x >= (1 << 63) else x


def _mix_py(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, workload: int, tensor: int) -> int:
    """64-bit key of one tensor's counter stream."""
    return _mix_py((seed << 32) ^ (workload << 8) ^ tensor ^ 0x5DEECE66D)


def _srl(z: torch.Tensor, k: int) -> torch.Tensor:
    # logical right shift on int64 (torch's >> is arithmetic)
    return (z >> k) & ((1 << (64 - k)) - 1)


def bits64(key: int, idx: torch.Tensor) -> torch.Tensor:
    """SplitMix64 counter outputs for int64 counters ``idx`` (any device)."""
    z = idx.to(torch.int64) + 1
    z = z * _to_i64(_GAMMA) + _to_i64(key)
    z = (z ^ _srl(z, 30)) * _to_i64(_M1)
    z = (z ^ _srl(z, 27)) * _to_i64(_M2)
    return z ^ _srl(z, 31)


def uniform(key: int, idx: torch.Tensor) -> torch.Tensor:
    """float64 uniforms strictly inside (0, 1)."""
    b = _srl(bits64(key, idx), 11)
    return (b.to(torch.float64) + 0.5) * (1.0 / 9007199254740992.0)


def normal(key: int, idx: torch.Tensor) -> torch.Tensor:
    """float64 N(0,1) draws, one per counter in ``idx`` (Box-Muller)."""
    i2 = idx.to(torch.int64) * 2
    u1 = uniform(key, i2)
    u2 = uniform(key, i2 + 1)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


def round_to(x64: torch.Tensor, dtype: torch.dtype) -> torch.Tensor:
    """Single rounding of float64 values to the storage dtype (RNE)."""
    if dtype == torch.bfloat16:
        # float64 -> float32 first is exact for our ranges except for the
        # mantissa bits below fp32's, which a direct RNE to bf16 would also
        # consider; do a direct round from the fp64 bit pattern instead.
        return _f64_to_bf16_rne(x64)
    return x64.to(dtype)


def _f64_to_bf16_rne(x64: torch.Tensor) -> torch.Tensor:
    """Round float64 straight to bf16 (round to nearest, ties to even).

    bf16 keeps the top 16 bits of an fp32 pattern. Rounding fp64 -> fp32 -> bf16
    could double-round; rounding directly on the fp64 mantissa avoids it.
    Finite inputs only (our draws are bounded by about 9 in magnitude).
    """
    b = x64.contiguous().view(torch.int64)
    # fp64 has 52 fraction bits, bf16 has 7: drop 45 bits with RNE.
    lsb = _srl(b, 45) & 1
    rounded = b + ((1 << 44) - 1) + lsb
    rounded = rounded & ~((1 << 45) - 1)
    y = rounded.view(torch.float64)
    # y is now exactly representable in bf16 (or 0); these casts are exact
    return y.to(torch.float32).to(torch.bfloat16)


# --------------------------------------------------------------------------
# workloads


@dataclasses.dataclass(frozen=True)
class Workload:
    """One GDPA problem family: shapes, activation, scale, input recipe."""
    wid: int
    name: str
    dtype: torch.dtype
    phi: int
    B: int
    h: int
    dh: int
    m: int
    lengths: str            # "fixed:n" | "uniform:lo:hi" | "powerlaw:alpha:lo:hi"
    qk_std: str             # "1" or "rsqrt_dh"
    kv_recipe: str          # "normal" | "linear_map"
    backward: bool
    scale: float

    @property
    def phi_name(self) -> str:
        return PHI_NAMES[self.phi]


def _wl(wid, name, dtype, phi, B, h, dh, m, lengths, qk_std, kv_recipe, backward):
    scale = 1.0 / math.sqrt(dh) if phi == PHI_SOFTMAX else 1.0
    return Workload(wid, name, dtype, phi, B, h, dh, m, lengths, qk_std, kv_recipe,
                    backward, scale)


WORKLOADS: Dict[int, Workload] = {
    1: _wl(1, "gdpa_fwd_f32_silu_B4_n64_h2_dh32_m64", torch.float32, PHI_SILU,
           4, 2, 32, 64, "fixed:64", "rsqrt_dh", "normal", False),
    2: _wl(2, "gdpa_fwd_bf16_silu_B256_n512_h4_dh64_m256", torch.bfloat16, PHI_SILU,
           256, 4, 64, 256, "fixed:512", "1", "linear_map", False),
    3: _wl(3, "gdpa_fwd_bf16_softmax_B512_nU16-2048_h8_dh64_m512", torch.bfloat16,
           PHI_SOFTMAX, 512, 8, 64, 512, "uniform:16:2048", "1", "normal", False),
    4: _wl(4, "gdpa_fwdbwd_bf16_silu_B512_nU64-1024_h8_dh128_m1024", torch.bfloat16,
           PHI_SILU, 512, 8, 128, 1024, "uniform:64:1024", "rsqrt_dh", "normal", True),
    5: _wl(5, "gdpa_fwdbwd_bf16_softmax_B1024_nPL1.5-32-4096_h16_dh64_m2048",
           torch.bfloat16, PHI_SOFTMAX, 1024, 16, 64, 2048, "powerlaw:1.5:32:4096", "1",
           "normal", True),
}


def lengths(wl: Workload, seed: int = 0) -> np.ndarray:
    """Per-sample history lengths n_b (int64 numpy array of size B)."""
    kind, *args = wl.lengths.split(":")
    if kind == "fixed":
        return np.full(wl.B, int(args[0]), dtype=np.int64)
    u = uniform(stream_key(seed, wl.wid, T_LENGTHS),
                torch.arange(wl.B, dtype=torch.int64)).numpy()
    if kind == "uniform":
        lo, hi = int(args[0]), int(args[1])
        n = lo + np.floor(u * (hi - lo + 1)).astype(np.int64)
        return np.minimum(n, hi)
    if kind == "powerlaw":
        alpha, lo, hi = float(args[0]), int(args[1]), int(args[2])
        support = np.arange(lo, hi + 1, dtype=np.float64)
        pmf = support ** (-alpha)
        cdf = np.cumsum(pmf)
        cdf /= cdf[-1]
        idx = np.searchsorted(cdf, u, side="left")
        return (lo + np.minimum(idx, hi - lo)).astype(np.int64)
    raise ValueError(wl.lengths)


def offsets_from_lengths(n: Sequence[int]) -> np.ndarray:
    off = np.zeros(len(n) + 1, dtype=np.int64)
    off[1:] = np.cumsum(np.asarray(n, dtype=np.int64))
    return off


def _std(wl: Workload, which: str) -> float:
    if which == "1":
        return 1.0
    if which == "rsqrt_dh":
        return 1.0 / math.sqrt(wl.dh)
    raise ValueError(which)


def _normal_block(key: int, start: int, count: int, device, chunk: int = 1 << 24):
    out = torch.empty(count, dtype=torch.float64, device=device)
    for c0 in range(0, count, chunk):
        c1 = min(count, c0 + chunk)
        idx = torch.arange(start + c0, start + c1, dtype=torch.int64, device=device)
        out[c0:c1] = normal(key, idx)
    return out


def _gen_rows(key, row_ranges, row_len, std, dtype, device, chunk: int = 1 << 24):
    """Rows [r0, r1) of a flat N(0, std^2) tensor with rows of ``row_len``.

    Written chunk by chunk into the storage dtype, so that no float64 copy of
    a large tensor is ever held.
    """
    total = sum(max(0, r1 - r0) for r0, r1 in row_ranges) * row_len
    out = torch.empty(total, dtype=dtype, device=device)
    pos = 0
    for r0, r1 in row_ranges:
        if r1 <= r0:
            continue
        start, count = r0 * row_len, (r1 - r0) * row_len
        for c0 in range(0, count, chunk):
            c1 = min(count, c0 + chunk)
            idx = torch.arange(start + c0, start + c1, dtype=torch.int64, device=device)
            out[pos + c0:pos + c1] = round_to(normal(key, idx) * std, dtype)
        pos += count
    return out


CTX_DIM = 64   # context vector length of the linear-map workload


def _wg_weight(wl: Workload, key_w: int, device) -> torch.Tensor:
    """fp32 weight [h*m*dh, 64] of the linear-map recipe, N(0, 1/(64 dh))."""
    rows = wl.h * wl.m * wl.dh
    wstd = 1.0 / math.sqrt(CTX_DIM * wl.dh)
    w = _normal_block(key_w, 0, rows * CTX_DIM, device).mul_(wstd)
    return w.to(torch.float32).view(rows, CTX_DIM)


def _wg_contexts(ctx_key: int, samples, device) -> torch.Tensor:
    """fp32 N(0, 1) context vectors [len(samples), 64], one per sample."""
    if not samples:
        return torch.empty(0, CTX_DIM, dtype=torch.float32, device=device)
    return torch.stack([_normal_block(ctx_key, b * CTX_DIM, CTX_DIM, device)
                        for b in samples]).to(torch.float32)


def weight_gen_factors(wid: int, which: str = "k", seed: int = 0, samples=None, device="cpu"):
    """The random numbers of the linear-map recipe: the fp32 weight [h*m*dh, 64]
    of K (``which="k"``) or V, and the fp32 contexts [len(samples), 64]."""
    wl = WORKLOADS[wid]
    sel = list(range(wl.B)) if samples is None else [int(b) for b in samples]
    key_w = stream_key(seed, wid, T_WK if which == "k" else T_WV)
    w = _wg_weight(wl, key_w, device)
    ctx = _wg_contexts(stream_key(seed, wid, T_CTX), sel, device)
    return w, ctx


def _linear_map_kv(wl: Workload, key_w: int, ctx_key: int, samples, dtype, device):
    """K_b = reshape(W c_b): fp32 weight [h*m*dh, 64], fp32 64-dim N(0,1) context
    (the workload's input recipe, evaluated in float64 and rounded once)."""
    w = _wg_weight(wl, key_w, device).to(torch.float64)
    out = [round_to(w @ c.to(torch.float64), dtype)
           for c in _wg_contexts(ctx_key, list(samples), device)]
    return torch.cat(out) if out else torch.empty(0, dtype=dtype, device=device)


def make_inputs(wid: int, device="cpu", seed: int = 0,
                samples: Optional[Iterable[int]] = None,
                backward: Optional[bool] = None,
                n_override: Optional[Sequence[int]] = None) -> dict:
    """Generate one workload's inputs (or the inputs of a subset of samples).

    Returns a dict with ``q [T,h,dh]``, ``k, v [B,h,m,dh]``, ``dout [T,h,dh]``
    (when the workload has a backward, or ``backward=True``), int64 numpy
    ``lengths`` and ``offsets``, and the workload.  With ``samples`` the batch
    holds only those samples (in that order), each bit-identical to its slice
    of the full batch.
    """
    wl = WORKLOADS[wid]
    n_all = np.asarray(n_override, dtype=np.int64) if n_override is not None \
        else lengths(wl, seed)
    off_all = offsets_from_lengths(n_all)
    sel = list(range(wl.B)) if samples is None else [int(b) for b in samples]
    n_sel = n_all[sel]
    hd = wl.h * wl.dh
    qrows = [(int(off_all[b]), int(off_all[b + 1])) for b in sel]
    T = int(n_sel.sum())
    std_qk = _std(wl, wl.qk_std)
    q = _gen_rows(stream_key(seed, wid, T_Q), qrows, hd, std_qk, wl.dtype, device)
    q = q.view(T, wl.h, wl.dh)
    kv_rows = [(b, b + 1) for b in sel]
    kv_len = wl.h * wl.m * wl.dh
    if wl.kv_recipe == "normal":
        k = _gen_rows(stream_key(seed, wid, T_K), kv_rows, kv_len, std_qk, wl.dtype, device)
        v = _gen_rows(stream_key(seed, wid, T_V), kv_rows, kv_len, std_qk, wl.dtype, device)
    else:
        ctx = stream_key(seed, wid, T_CTX)
        k = _linear_map_kv(wl, stream_key(seed, wid, T_WK), ctx, sel, wl.dtype, device)
        v = _linear_map_kv(wl, stream_key(seed, wid, T_WV), ctx, sel, wl.dtype, device)
    k = k.view(len(sel), wl.h, wl.m, wl.dh)
    v = v.view(len(sel), wl.h, wl.m, wl.dh)
    out = dict(workload=wl, q=q, k=k, v=v, lengths=n_sel,
               offsets=offsets_from_lengths(n_sel), samples=sel)
    want_bwd = wl.backward if backward is None else backward
    if want_bwd:
        d = _gen_rows(stream_key(seed, wid, T_DOUT), qrows, hd, 1.0, wl.dtype, device)
        out["dout"] = d.view(T, wl.h, wl.dh)
    return out


def random_problem(rng_seed: int, B: int, h: int, dh: int, m: int, n: Sequence[int],
                   dtype=torch.bfloat16, std: float = 1.0, device="cpu") -> dict:
    """Small ad-hoc jagged problem from the same generator (for edge cases)."""
    key_base = _mix_py(0xC0FFEE ^ (rng_seed << 20) ^ (B << 10) ^ (h << 5) ^ dh ^ (m << 40))
    n = np.asarray(n, dtype=np.int64)
    T = int(n.sum())

    def draw(tid, count):
        x = _normal_block(_mix_py(key_base ^ tid), 0, count, device)
        return round_to(x * std, dtype)

    return dict(q=draw(T_Q, T * h * dh).view(T, h, dh),
                k=draw(T_K, B * h * m * dh).view(B, h, m, dh),
                v=draw(T_V, B * h * m * dh).view(B, h, m, dh),
                dout=draw(T_DOUT, T * h * dh).view(T, h, dh),
                lengths=n, offsets=offsets_from_lengths(n))
