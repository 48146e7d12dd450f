"""GDPA oracle (plain fp64 C, OpenMP) and its ctypes loader.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
benchmark's CPU-baseline leg import this package.  The product library in
``recsys_context_personalised_b200`` never imports it, and the oracle shares
no code with the CUDA path.  The arithmetic lives in ``gdpa_oracle.c``; this
file only compiles it, marshals arrays and converts results.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdpa_oracle.c")
_LIB = os.path.join(_HERE, "libgdpa_oracle.so")
_lib = None

PHI = {"identity": 0, "silu": 1, "softmax": 2, "relu": 3, "gelu": 4}


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (IEEE double, no fast-math)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-fno-fast-math",
           "-ffp-contract=off", "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def load(path: str = None):
    global _lib
    if path is None and _lib is not None:
        return _lib
    lib = ctypes.CDLL(build() if path is None else path)
    i32, i64p, fp, dp, f64 = (ctypes.c_int, ctypes.POINTER(ctypes.c_int64),
                              ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_double),
                              ctypes.c_double)
    lib.gdpa_oracle_fwd.argtypes = [i32, i32, i32, i32, i64p, fp, fp, fp, i32, f64, dp, dp, i32]
    lib.gdpa_oracle_fwd.restype = i32
    lib.gdpa_oracle_bwd.argtypes = [i32, i32, i32, i32, i64p, fp, fp, fp, fp, i32, f64,
                                    dp, dp, dp, i32]
    lib.gdpa_oracle_bwd.restype = i32
    lib.gdpa_oracle_fwd_bias.argtypes = [i32, i32, i32, i32, i64p, fp, fp, fp, fp, fp, i32, f64,
                                         dp, dp, i32]
    lib.gdpa_oracle_fwd_bias.restype = i32
    lib.gdpa_oracle_bwd_bias.argtypes = [i32, i32, i32, i32, i64p, fp, fp, fp, fp, fp, i32, f64,
                                         dp, dp, dp, dp, dp, i32]
    lib.gdpa_oracle_bwd_bias.restype = i32
    lib.gdpa_oracle_max_threads.restype = i32
    if path is None:
        _lib = lib
    return lib


def _f32(x) -> np.ndarray:
    """Exact float32 copy of a bf16/fp32 torch tensor or numpy array."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().float().numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _phi(phi) -> int:
    return PHI[phi] if isinstance(phi, str) else int(phi)


def max_threads(lib=None) -> int:
    return (lib or load()).gdpa_oracle_max_threads()


def _opt(x, shape):
    """Exact float32 copy of an optional bias, checked against its shape."""
    if x is None:
        return None
    x = _f32(x)
    assert x.shape == shape, (x.shape, shape)
    return x


def _optp(x, ct):
    return None if x is None else _ptr(x, ct)


def fwd(q, k, v, offsets, phi, scale, nthreads: int = 0, lib=None, b1=None, b2=None):
    """O [T,h,dh] float64 and LSE [h,T] float64 (NaN-free only for softmax).

    ``b1`` [B,h,m] and ``b2`` [B,h,dh] are the optional biases of
    phi(s Q K^T + b1) V + b2."""
    lib = lib or load()
    q, k, v = _f32(q), _f32(k), _f32(v)
    off = np.ascontiguousarray(offsets, dtype=np.int64)
    B, h, m, dh = k.shape
    T = int(off[-1])
    assert q.shape == (T, h, dh) and v.shape == k.shape and off.shape == (B + 1,)
    b1, b2 = _opt(b1, (B, h, m)), _opt(b2, (B, h, dh))
    o = np.zeros((T, h, dh), dtype=np.float64)
    lse = np.zeros((h, T), dtype=np.float64)
    rc = lib.gdpa_oracle_fwd_bias(B, h, dh, m, _ptr(off, ctypes.c_int64),
                                  _ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                  _ptr(v, ctypes.c_float), _optp(b1, ctypes.c_float),
                                  _optp(b2, ctypes.c_float), _phi(phi), float(scale),
                                  _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double),
                                  int(nthreads))
    if rc != 0:
        raise RuntimeError(f"gdpa_oracle_fwd failed with code {rc}")
    return o, lse


def bwd(q, k, v, dout, offsets, phi, scale, nthreads: int = 0, lib=None, b1=None,
        bias_grads: bool = False):
    """(dQ [T,h,dh], dK [B,h,m,dh], dV [B,h,m,dh]) in float64, and with
    ``bias_grads`` also (dB1 [B,h,m], dB2 [B,h,dh]).  ``b1`` is the optional
    key bias (the output bias b2 does not enter the gradients)."""
    lib = lib or load()
    q, k, v, g = _f32(q), _f32(k), _f32(v), _f32(dout)
    off = np.ascontiguousarray(offsets, dtype=np.int64)
    B, h, m, dh = k.shape
    T = int(off[-1])
    assert q.shape == (T, h, dh) and g.shape == q.shape and v.shape == k.shape
    b1 = _opt(b1, (B, h, m))
    dq = np.zeros((T, h, dh), dtype=np.float64)
    dk = np.zeros((B, h, m, dh), dtype=np.float64)
    dv = np.zeros((B, h, m, dh), dtype=np.float64)
    db1 = np.zeros((B, h, m), dtype=np.float64) if bias_grads else None
    db2 = np.zeros((B, h, dh), dtype=np.float64) if bias_grads else None
    rc = lib.gdpa_oracle_bwd_bias(B, h, dh, m, _ptr(off, ctypes.c_int64),
                                  _ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                  _ptr(v, ctypes.c_float), _optp(b1, ctypes.c_float),
                                  _ptr(g, ctypes.c_float), _phi(phi), float(scale),
                                  _ptr(dq, ctypes.c_double), _ptr(dk, ctypes.c_double),
                                  _ptr(dv, ctypes.c_double), _optp(db1, ctypes.c_double),
                                  _optp(db2, ctypes.c_double), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"gdpa_oracle_bwd failed with code {rc}")
    if bias_grads:
        return dq, dk, dv, db1, db2
    return dq, dk, dv


# --------------------------------------------------------------------------
# Weight Generation (context vector -> per-sample K or V), weight_gen_oracle.c

_WG_SRC = os.path.join(_HERE, "weight_gen_oracle.c")
_WG_LIB = os.path.join(_HERE, "libwg_oracle.so")
_wg_lib = None


def wg_load(path: str = None):
    """Load (building if needed) the Weight Generation oracle library."""
    global _wg_lib
    if path is None and _wg_lib is not None:
        return _wg_lib
    lib = ctypes.CDLL(build(src=_WG_SRC, out=_WG_LIB) if path is None else path)
    i32, i64, fp, dp = ctypes.c_int, ctypes.c_int64, ctypes.POINTER(ctypes.c_float), \
        ctypes.POINTER(ctypes.c_double)
    lib.wg_oracle_fwd.argtypes = [i32, i64, i32, fp, fp, dp, i32]
    lib.wg_oracle_fwd.restype = i32
    lib.wg_oracle_bwd.argtypes = [i32, i64, i32, fp, fp, fp, dp, dp, i32]
    lib.wg_oracle_bwd.restype = i32
    if path is None:
        _wg_lib = lib
    return lib


def weight_gen(w, ctx, nthreads: int = 0, lib=None):
    """Y [B, F] float64 = ctx [B, C] applied to W [F, C]: Y[b, f] = sum_c W[f, c] ctx[b, c]."""
    lib = lib or wg_load()
    w, ctx = _f32(w), _f32(ctx)
    F, C = w.shape
    B = ctx.shape[0]
    assert ctx.shape == (B, C)
    y = np.zeros((B, F), dtype=np.float64)
    rc = lib.wg_oracle_fwd(B, F, C, _ptr(w, ctypes.c_float), _ptr(ctx, ctypes.c_float),
                           _ptr(y, ctypes.c_double), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"wg_oracle_fwd failed with code {rc}")
    return y


def weight_gen_bwd(w, ctx, dy, nthreads: int = 0, lib=None):
    """(dW [F, C], dctx [B, C]) float64 for an upstream dY [B, F]."""
    lib = lib or wg_load()
    w, ctx, dy = _f32(w), _f32(ctx), _f32(dy)
    F, C = w.shape
    B = ctx.shape[0]
    assert dy.shape == (B, F)
    dw = np.zeros((F, C), dtype=np.float64)
    dctx = np.zeros((B, C), dtype=np.float64)
    rc = lib.wg_oracle_bwd(B, F, C, _ptr(w, ctypes.c_float), _ptr(ctx, ctypes.c_float),
                           _ptr(dy, ctypes.c_float), _ptr(dw, ctypes.c_double),
                           _ptr(dctx, ctypes.c_double), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"wg_oracle_bwd failed with code {rc}")
    return dw, dctx


# --------------------------------------------------------------------------
# seed-query attention pooling (first level of HSP), pooling_oracle.c

_POOL_SRC = os.path.join(_HERE, "pooling_oracle.c")
_POOL_LIB = os.path.join(_HERE, "libpool_oracle.so")
_pool_lib = None


def pool_load(path: str = None):
    """Load (building if needed) the pooling oracle library."""
    global _pool_lib
    if path is None and _pool_lib is not None:
        return _pool_lib
    lib = ctypes.CDLL(build(src=_POOL_SRC, out=_POOL_LIB) if path is None else path)
    i32, i64p, fp, dp, f64 = (ctypes.c_int, ctypes.POINTER(ctypes.c_int64),
                              ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_double),
                              ctypes.c_double)
    lib.pool_oracle_fwd.argtypes = [i32, i32, i32, i32, i64p, fp, fp, fp, f64, dp, dp, i32]
    lib.pool_oracle_fwd.restype = i32
    lib.pool_oracle_bwd.argtypes = [i32, i32, i32, i32, i64p, fp, fp, fp, fp, f64, dp, dp, dp,
                                    i32]
    lib.pool_oracle_bwd.restype = i32
    if path is None:
        _pool_lib = lib
    return lib


def pool_fwd(seeds, k, v, offsets, scale, nthreads: int = 0, lib=None):
    """(O [B, h, S, dh], LSE [B, h, S]) float64 of seed-query attention pooling."""
    lib = lib or pool_load()
    seeds, k, v = _f32(seeds), _f32(k), _f32(v)
    off = np.ascontiguousarray(offsets, dtype=np.int64)
    h, S, dh = seeds.shape
    B = off.shape[0] - 1
    assert k.shape == (int(off[-1]), h, dh) and v.shape == k.shape
    o = np.zeros((B, h, S, dh), dtype=np.float64)
    lse = np.zeros((B, h, S), dtype=np.float64)
    rc = lib.pool_oracle_fwd(B, h, dh, S, _ptr(off, ctypes.c_int64), _ptr(seeds, ctypes.c_float),
                             _ptr(k, ctypes.c_float), _ptr(v, ctypes.c_float), float(scale),
                             _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"pool_oracle_fwd failed with code {rc}")
    return o, lse


def pool_bwd(seeds, k, v, dout, offsets, scale, nthreads: int = 0, lib=None):
    """(dseeds [h, S, dh], dK [T, h, dh], dV [T, h, dh]) float64."""
    lib = lib or pool_load()
    seeds, k, v, g = _f32(seeds), _f32(k), _f32(v), _f32(dout)
    off = np.ascontiguousarray(offsets, dtype=np.int64)
    h, S, dh = seeds.shape
    B = off.shape[0] - 1
    assert g.shape == (B, h, S, dh)
    ds = np.zeros((h, S, dh), dtype=np.float64)
    dk = np.zeros(k.shape, dtype=np.float64)
    dv = np.zeros(v.shape, dtype=np.float64)
    rc = lib.pool_oracle_bwd(B, h, dh, S, _ptr(off, ctypes.c_int64), _ptr(seeds, ctypes.c_float),
                             _ptr(k, ctypes.c_float), _ptr(v, ctypes.c_float),
                             _ptr(g, ctypes.c_float), float(scale), _ptr(ds, ctypes.c_double),
                             _ptr(dk, ctypes.c_double), _ptr(dv, ctypes.c_double), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"pool_oracle_bwd failed with code {rc}")
    return ds, dk, dv


# --------------------------------------------------------------------------
# sliding-window self-attention on the jagged sequence, window_oracle.c

_WIN_SRC = os.path.join(_HERE, "window_oracle.c")
_WIN_LIB = os.path.join(_HERE, "libwin_oracle.so")
_win_lib = None


def win_load(path: str = None):
    """Load (building if needed) the sliding-window oracle library."""
    global _win_lib
    if path is None and _win_lib is not None:
        return _win_lib
    lib = ctypes.CDLL(build(src=_WIN_SRC, out=_WIN_LIB) if path is None else path)
    i32, i64p, fp, dp, f64 = (ctypes.c_int, ctypes.POINTER(ctypes.c_int64),
                              ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_double),
                              ctypes.c_double)
    lib.win_oracle_fwd.argtypes = [i32, i32, i32, i32, i64p, fp, fp, fp, f64, dp, dp, i32]
    lib.win_oracle_fwd.restype = i32
    lib.win_oracle_bwd.argtypes = [i32, i32, i32, i32, i64p, fp, fp, fp, fp, f64, dp, dp, dp, i32]
    lib.win_oracle_bwd.restype = i32
    if path is None:
        _win_lib = lib
    return lib


def win_fwd(q, k, v, offsets, window, scale, nthreads: int = 0, lib=None):
    """(O [T, h, dh], LSE [h, T]) float64 of causal sliding-window attention."""
    lib = lib or win_load()
    q, k, v = _f32(q), _f32(k), _f32(v)
    off = np.ascontiguousarray(offsets, dtype=np.int64)
    T, h, dh = q.shape
    B = off.shape[0] - 1
    assert k.shape == q.shape and v.shape == q.shape and int(off[-1]) == T
    o = np.zeros((T, h, dh), dtype=np.float64)
    lse = np.zeros((h, T), dtype=np.float64)
    rc = lib.win_oracle_fwd(B, h, dh, int(window), _ptr(off, ctypes.c_int64),
                            _ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                            _ptr(v, ctypes.c_float), float(scale), _ptr(o, ctypes.c_double),
                            _ptr(lse, ctypes.c_double), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"win_oracle_fwd failed with code {rc}")
    return o, lse


def win_bwd(q, k, v, dout, offsets, window, scale, nthreads: int = 0, lib=None):
    """(dQ, dK, dV) [T, h, dh] float64."""
    lib = lib or win_load()
    q, k, v, g = _f32(q), _f32(k), _f32(v), _f32(dout)
    off = np.ascontiguousarray(offsets, dtype=np.int64)
    T, h, dh = q.shape
    B = off.shape[0] - 1
    dq, dk, dv = (np.zeros((T, h, dh), dtype=np.float64) for _ in range(3))
    rc = lib.win_oracle_bwd(B, h, dh, int(window), _ptr(off, ctypes.c_int64),
                            _ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                            _ptr(v, ctypes.c_float), _ptr(g, ctypes.c_float), float(scale),
                            _ptr(dq, ctypes.c_double), _ptr(dk, ctypes.c_double),
                            _ptr(dv, ctypes.c_double), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"win_oracle_bwd failed with code {rc}")
    return dq, dk, dv
