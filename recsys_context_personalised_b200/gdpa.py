"""ctypes binding of libgdpa.so (the C ABI declared in include/gdpa.h).

Argument marshalling only: every step of GDPA runs in the library's CUDA
kernels.  PyTorch provides device memory and the current CUDA stream.  There
is no CPU fallback: if the shared library is missing or fails to load, every
call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdpa.so")

PHI_IDENTITY, PHI_SILU, PHI_SOFTMAX, PHI_RELU, PHI_GELU = 0, 1, 2, 3, 4
PHI = {"identity": PHI_IDENTITY, "silu": PHI_SILU, "softmax": PHI_SOFTMAX, "relu": PHI_RELU,
       "gelu": PHI_GELU}
DTYPE_F32, DTYPE_BF16 = 0, 1
STATUS = {0: "GDPA_OK", 1: "GDPA_ERR_INVALID_ARG", 2: "GDPA_ERR_UNSUPPORTED",
          3: "GDPA_ERR_CUDA", 4: "GDPA_ERR_TIMEOUT", 5: "GDPA_ERR_WORKSPACE"}

EXPORTED = ("gdpa_fwd_workspace_size", "gdpa_bwd_workspace_size", "gdpa_fwd", "gdpa_bwd",
            "gdpa_workspace_status", "gdpa_fwd_bias", "gdpa_bwd_bias", "gdpa_weight_gen",
            "gdpa_status_string",
            "gdpa_last_launch_count", "gdpa_timing_enable", "gdpa_timing_read")


class Problem(ctypes.Structure):
    """Mirror of gdpa_problem_t."""
    _fields_ = [("B", ctypes.c_int32), ("h", ctypes.c_int32), ("dh", ctypes.c_int32),
                ("m", ctypes.c_int32), ("max_n", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("total_tokens", ctypes.c_int64), ("phi", ctypes.c_int32),
                ("scale", ctypes.c_float)]


class KernelTime(ctypes.Structure):
    """Mirror of gdpa_kernel_time_t."""
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int32),
                ("total_ms", ctypes.c_float)]


class GdpaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code


_lib = None


def load(path: str = LIB_PATH):
    """Load libgdpa.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libgdpa.so not built at {path}; run __graft_entry__.build()")
    lib = ctypes.CDLL(path)
    vp, sz, pp = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(Problem)
    lib.gdpa_fwd_workspace_size.argtypes = [pp, ctypes.POINTER(sz)]
    lib.gdpa_bwd_workspace_size.argtypes = [pp, ctypes.POINTER(sz)]
    lib.gdpa_fwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.gdpa_bwd.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.gdpa_workspace_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int32)]
    lib.gdpa_fwd_bias.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.gdpa_bwd_bias.argtypes = [pp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                  sz, vp]
    lib.gdpa_status_string.argtypes = [ctypes.c_int]
    lib.gdpa_status_string.restype = ctypes.c_char_p
    lib.gdpa_last_launch_count.restype = ctypes.c_int32
    lib.gdpa_timing_enable.argtypes = [ctypes.c_int32]
    lib.gdpa_timing_enable.restype = ctypes.c_int
    lib.gdpa_timing_read.argtypes = [ctypes.POINTER(KernelTime), ctypes.c_int32]
    lib.gdpa_timing_read.restype = ctypes.c_int32
    lib.gdpa_weight_gen.argtypes = [ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, vp, vp, vp,
                                    vp, vp]
    lib.gdpa_weight_gen_bwd_workspace_size.argtypes = [ctypes.c_int32, ctypes.c_int64,
                                                       ctypes.c_int32, ctypes.POINTER(sz)]
    lib.gdpa_weight_gen_bwd_workspace_size.restype = ctypes.c_int
    lib.gdpa_weight_gen_bwd.argtypes = [ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, vp, vp,
                                        vp, vp, vp, vp, sz, vp]
    lib.gdpa_weight_gen_bwd.restype = ctypes.c_int
    i32 = ctypes.c_int32
    lib.gdpa_pool_workspace_size.argtypes = [i32, i32, i32, i32, ctypes.POINTER(sz)]
    lib.gdpa_pool_workspace_size.restype = ctypes.c_int
    lib.gdpa_pool_fwd.argtypes = [i32, i32, i32, i32, ctypes.c_int64, i32, ctypes.c_float, vp, vp,
                                  vp, vp, vp, vp, vp, sz, vp]
    lib.gdpa_pool_fwd.restype = ctypes.c_int
    lib.gdpa_window_workspace_size.argtypes = [i32, i32, i32, ctypes.c_int64, ctypes.POINTER(sz)]
    lib.gdpa_window_workspace_size.restype = ctypes.c_int
    lib.gdpa_window_fwd.argtypes = [i32, i32, i32, ctypes.c_int64, i32, i32, ctypes.c_float, vp,
                                    vp, vp, vp, vp, vp, vp, sz, vp]
    lib.gdpa_window_fwd.restype = ctypes.c_int
    i64, f32 = ctypes.c_int64, ctypes.c_float
    lib.gdpa_pool_bwd_workspace_size.argtypes = [i32, i32, i32, i32, i64, ctypes.POINTER(sz)]
    lib.gdpa_pool_bwd_workspace_size.restype = ctypes.c_int
    lib.gdpa_pool_bwd.argtypes = [i32, i32, i32, i32, i64, i32, f32] + [vp] * 11 + [sz, vp]
    lib.gdpa_pool_bwd.restype = ctypes.c_int
    lib.gdpa_window_bwd_workspace_size.argtypes = [i32, i32, i32, i64, ctypes.POINTER(sz)]
    lib.gdpa_window_bwd_workspace_size.restype = ctypes.c_int
    lib.gdpa_window_bwd.argtypes = [i32, i32, i32, i64, i32, i32, f32] + [vp] * 11 + [sz, vp]
    lib.gdpa_window_bwd.restype = ctypes.c_int
    for name in EXPORTED[:8]:
        getattr(lib, name).restype = ctypes.c_int
    if path == LIB_PATH:
        _lib = lib
    return lib


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def problem(B: int, h: int, dh: int, m: int, total_tokens: int, max_n: int, phi, scale: float,
            dtype: torch.dtype) -> Problem:
    phi = PHI[phi] if isinstance(phi, str) else int(phi)
    dt = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}.get(dtype, -1)
    return Problem(B, h, dh, m, max_n, dt, total_tokens, phi, scale)


def problem_for(q: torch.Tensor, k: torch.Tensor, offsets_host, phi, scale: float,
                max_n: Optional[int] = None) -> Problem:
    """Problem of a batch; ``offsets_host`` is a host sequence (for T and max_n)."""
    B, h, m, dh = k.shape
    off = [int(x) for x in offsets_host]
    T = off[-1]
    if max_n is None:
        max_n = max((off[i + 1] - off[i] for i in range(B)), default=0)
    return problem(B, h, dh, m, T, max_n, phi, scale, q.dtype)


def fwd_workspace_bytes(p: Problem) -> int:
    n = ctypes.c_size_t()
    rc = load().gdpa_fwd_workspace_size(ctypes.byref(p), ctypes.byref(n))
    if rc:
        raise GdpaError(rc, "gdpa_fwd_workspace_size")
    return n.value


def bwd_workspace_bytes(p: Problem) -> int:
    n = ctypes.c_size_t()
    rc = load().gdpa_bwd_workspace_size(ctypes.byref(p), ctypes.byref(n))
    if rc:
        raise GdpaError(rc, "gdpa_bwd_workspace_size")
    return n.value


def workspace(nbytes: int, device) -> torch.Tensor:
    """A 256-byte aligned device buffer (torch's caching allocator aligns to 512)."""
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def fwd(p: Problem, q, offsets, k, v, o=None, lse=None, ws=None, stream=None
        ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Run gdpa_fwd; allocates the outputs/workspace with torch when not given."""
    lib = load()
    if o is None:
        o = torch.empty_like(q)
    if lse is None and p.phi == PHI_SOFTMAX:
        lse = torch.empty((p.h, p.total_tokens), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(fwd_workspace_bytes(p), q.device)
    rc = lib.gdpa_fwd(ctypes.byref(p), _ptr(q), _ptr(offsets), _ptr(k), _ptr(v), _ptr(o),
                      _ptr(lse), _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise GdpaError(rc, "gdpa_fwd")
    return o, lse


def bwd(p: Problem, q, offsets, k, v, o, lse, dout, dq=None, dk=None, dv=None, ws=None,
        stream=None):
    """Run gdpa_bwd; returns (dq, dk, dv)."""
    lib = load()
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if ws is None:
        ws = workspace(bwd_workspace_bytes(p), q.device)
    rc = lib.gdpa_bwd(ctypes.byref(p), _ptr(q), _ptr(offsets), _ptr(k), _ptr(v), _ptr(o),
                      _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(),
                      _stream(stream))
    if rc:
        raise GdpaError(rc, "gdpa_bwd")
    return dq, dk, dv


def fwd_bias(p: Problem, q, offsets, k, v, b1=None, b2=None, o=None, lse=None, ws=None,
             stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Run gdpa_fwd_bias: o = phi(s q k^T + b1) v + b2 (fp32 biases b1 [B,h,m],
    b2 [B,h,dh], either may be None)."""
    lib = load()
    if o is None:
        o = torch.empty_like(q)
    if lse is None and p.phi == PHI_SOFTMAX:
        lse = torch.empty((p.h, p.total_tokens), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(fwd_workspace_bytes(p), q.device)
    rc = lib.gdpa_fwd_bias(ctypes.byref(p), _ptr(q), _ptr(offsets), _ptr(k), _ptr(v), _ptr(b1),
                           _ptr(b2), _ptr(o), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise GdpaError(rc, "gdpa_fwd_bias")
    return o, lse


def bwd_bias(p: Problem, q, offsets, k, v, b1, b2, o, lse, dout, dq=None, dk=None, dv=None,
             db1=None, db2=None, want_bias_grads=True, ws=None, stream=None):
    """Run gdpa_bwd_bias; returns (dq, dk, dv, db1, db2) (the last two None
    when ``want_bias_grads`` is False and none were given)."""
    lib = load()
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if want_bias_grads:
        B, h, m, dh = k.shape
        db1 = torch.empty((B, h, m), dtype=torch.float32, device=k.device) if db1 is None else db1
        db2 = torch.empty((B, h, dh), dtype=torch.float32, device=k.device) if db2 is None else db2
    if ws is None:
        ws = workspace(bwd_workspace_bytes(p), q.device)
    rc = lib.gdpa_bwd_bias(ctypes.byref(p), _ptr(q), _ptr(offsets), _ptr(k), _ptr(v), _ptr(b1),
                           _ptr(b2), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                           _ptr(db1), _ptr(db2), _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise GdpaError(rc, "gdpa_bwd_bias")
    return dq, dk, dv, db1, db2


def weight_gen(w: torch.Tensor, ctx: torch.Tensor, y: Optional[torch.Tensor] = None,
               status_ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Run gdpa_weight_gen: y [B, F] bf16 = ctx [B, C] applied to w [F, C] (fp32)."""
    F, C = w.shape
    B = ctx.shape[0]
    if y is None:
        y = torch.empty((B, F), dtype=torch.bfloat16, device=w.device)
    rc = load().gdpa_weight_gen(B, F, C, _ptr(w), _ptr(ctx), _ptr(y), _ptr(status_ws),
                                _stream(stream))
    if rc:
        raise GdpaError(rc, "gdpa_weight_gen")
    return y


def weight_gen_bwd(w: torch.Tensor, ctx: torch.Tensor, dy: torch.Tensor, ws=None, stream=None):
    """Run gdpa_weight_gen_bwd; returns (dw [F, C], dctx [B, C]) in fp32."""
    lib = load()
    F, C = w.shape
    B = ctx.shape[0]
    n = ctypes.c_size_t()
    rc = lib.gdpa_weight_gen_bwd_workspace_size(B, F, C, ctypes.byref(n))
    if rc:
        raise GdpaError(rc, "gdpa_weight_gen_bwd_workspace_size")
    if ws is None:
        ws = workspace(n.value, w.device)
    dw = torch.empty((F, C), dtype=torch.float32, device=w.device)
    dctx = torch.empty((B, C), dtype=torch.float32, device=w.device)
    rc = lib.gdpa_weight_gen_bwd(B, F, C, _ptr(w), _ptr(ctx), _ptr(dy), _ptr(dw), _ptr(dctx),
                                 _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise GdpaError(rc, "gdpa_weight_gen_bwd")
    return dw, dctx


def _batch_shape(offsets_host, shape):
    """(B, T, max_n) of a jagged batch: from ``shape`` when given, else from
    the host copy of the offsets."""
    if shape is not None:
        return tuple(int(x) for x in shape)
    off = [int(x) for x in offsets_host]
    B = len(off) - 1
    return B, off[-1], max((off[i + 1] - off[i] for i in range(B)), default=0)


def pool_fwd(seeds: torch.Tensor, offsets, k: torch.Tensor, v: torch.Tensor, scale: float,
             offsets_host, o=None, lse=None, ws=None, stream=None, want_lse=True, shape=None):
    """Run gdpa_pool_fwd (seed-query attention pooling): seeds [h, S, dh],
    jagged k, v [T, h, dh] with device ``offsets`` (host copy ``offsets_host``
    for B, T and max_n, or ``shape`` = (B, T, max_n)); returns
    (o [B, h, S, dh], lse [B, h, S] or None)."""
    lib = load()
    h, S, dh = seeds.shape
    B, T, max_n = _batch_shape(offsets_host, shape)
    if o is None:
        o = torch.empty((B, h, S, dh), dtype=seeds.dtype, device=seeds.device)
    if lse is None and want_lse:
        lse = torch.empty((B, h, S), dtype=torch.float32, device=seeds.device)
    if ws is None:
        n = ctypes.c_size_t()
        rc = lib.gdpa_pool_workspace_size(B, h, dh, S, ctypes.byref(n))
        if rc:
            raise GdpaError(rc, "gdpa_pool_workspace_size")
        ws = workspace(n.value, seeds.device)
    rc = lib.gdpa_pool_fwd(B, h, dh, S, T, max_n, scale, _ptr(seeds), _ptr(offsets), _ptr(k),
                           _ptr(v), _ptr(o), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise GdpaError(rc, "gdpa_pool_fwd")
    return o, lse


def window_fwd(q: torch.Tensor, offsets, k: torch.Tensor, v: torch.Tensor, window: int,
               scale: float, offsets_host, o=None, lse=None, ws=None, stream=None,
               want_lse=True, shape=None):
    """Run gdpa_window_fwd (causal sliding-window attention on jagged q, k, v
    [T, h, dh]; B and max_n from ``offsets_host`` or ``shape`` = (B, T, max_n));
    returns (o [T, h, dh], lse [h, T] or None)."""
    lib = load()
    T, h, dh = q.shape
    B, _, max_n = _batch_shape(offsets_host, shape)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((h, T), dtype=torch.float32, device=q.device)
    if ws is None:
        n = ctypes.c_size_t()
        rc = lib.gdpa_window_workspace_size(B, h, dh, T, ctypes.byref(n))
        if rc:
            raise GdpaError(rc, "gdpa_window_workspace_size")
        ws = workspace(n.value, q.device)
    rc = lib.gdpa_window_fwd(B, h, dh, T, max_n, window, scale, _ptr(q), _ptr(offsets), _ptr(k),
                             _ptr(v), _ptr(o), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise GdpaError(rc, "gdpa_window_fwd")
    return o, lse


def pool_bwd(seeds: torch.Tensor, offsets, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
             lse: torch.Tensor, dout: torch.Tensor, scale: float, offsets_host, dk=None, dv=None,
             dseeds=None, ws=None, stream=None, shape=None):
    """Run gdpa_pool_bwd: gradients of gdpa_pool_fwd for dout [B, h, S, dh];
    returns (dseeds fp32 [h, S, dh], dk, dv bf16 [T, h, dh])."""
    lib = load()
    h, S, dh = seeds.shape
    B, T, max_n = _batch_shape(offsets_host, shape)
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if dseeds is None:
        dseeds = torch.empty((h, S, dh), dtype=torch.float32, device=seeds.device)
    if ws is None:
        n = ctypes.c_size_t()
        rc = lib.gdpa_pool_bwd_workspace_size(B, h, dh, S, T, ctypes.byref(n))
        if rc:
            raise GdpaError(rc, "gdpa_pool_bwd_workspace_size")
        ws = workspace(n.value, seeds.device)
    rc = lib.gdpa_pool_bwd(B, h, dh, S, T, max_n, scale, _ptr(seeds), _ptr(offsets), _ptr(k),
                           _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dseeds), _ptr(dk),
                           _ptr(dv), _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise GdpaError(rc, "gdpa_pool_bwd")
    return dseeds, dk, dv


def window_bwd(q: torch.Tensor, offsets, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
               lse: torch.Tensor, dout: torch.Tensor, window: int, scale: float, offsets_host,
               dq=None, dk=None, dv=None, ws=None, stream=None, shape=None):
    """Run gdpa_window_bwd: gradients of gdpa_window_fwd for dout [T, h, dh];
    returns (dq, dk, dv) bf16 [T, h, dh]."""
    lib = load()
    T, h, dh = q.shape
    B, _, max_n = _batch_shape(offsets_host, shape)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if ws is None:
        n = ctypes.c_size_t()
        rc = lib.gdpa_window_bwd_workspace_size(B, h, dh, T, ctypes.byref(n))
        if rc:
            raise GdpaError(rc, "gdpa_window_bwd_workspace_size")
        ws = workspace(n.value, q.device)
    rc = lib.gdpa_window_bwd(B, h, dh, T, max_n, window, scale, _ptr(q), _ptr(offsets), _ptr(k),
                             _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                             _ptr(dv), _ptr(ws), ws.numel(), _stream(stream))
    if rc:
        raise GdpaError(rc, "gdpa_window_bwd")
    return dq, dk, dv


def workspace_status(ws: torch.Tensor, stream=None) -> int:
    """Device-detected status of the last call that used ``ws`` (synchronises)."""
    out = ctypes.c_int32()
    rc = load().gdpa_workspace_status(_ptr(ws), _stream(stream), ctypes.byref(out))
    if rc:
        raise GdpaError(rc, "gdpa_workspace_status")
    return out.value


def last_launch_count() -> int:
    return load().gdpa_last_launch_count()


def status_string(code: int) -> str:
    return load().gdpa_status_string(code).decode()


def timing_enable(on: bool = True) -> None:
    """Bracket every later kernel launch on this thread with CUDA events."""
    rc = load().gdpa_timing_enable(1 if on else 0)
    if rc:
        raise GdpaError(rc, "gdpa_timing_enable")


def timing_read() -> dict:
    """{kernel name: (launches, total ms)} since timing_enable(True); clears."""
    cap = 32
    buf = (KernelTime * cap)()
    n = load().gdpa_timing_read(buf, cap)
    if n < 0:
        raise GdpaError(3, "gdpa_timing_read")
    return {buf[i].name.decode(): (buf[i].launches, buf[i].total_ms) for i in range(min(n, cap))}
