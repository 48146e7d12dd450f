"""The C ABI library: loads, exports what include/gdpa.h declares, validates
arguments on the host (CPU only: no call here reaches a kernel launch)."""
import ctypes
import os
import re

import pytest
import torch

import recsys_context_personalised_b200 as pkg
from recsys_context_personalised_b200 import gdpa as G

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "gdpa.h")).read()
    return re.findall(r"GDPA_API\s+[\w\s\*]+?\b(gdpa_\w+)\s*\(", src)


def test_library_exports_every_declared_symbol():
    lib = pkg.load()
    names = _declared()
    assert set(G.EXPORTED) <= set(names) | {"gdpa_last_launch_count"}
    for n in names:
        assert hasattr(lib, n), n


def test_library_is_sm100a_and_in_tree():
    assert os.path.dirname(G.LIB_PATH) == os.path.join(ROOT, "recsys_context_personalised_b200")
    assert os.path.exists(G.LIB_PATH)


def test_status_strings():
    for code, name in G.STATUS.items():
        assert G.status_string(code).startswith(name)


def _p(**kw):
    base = dict(B=4, h=2, dh=64, m=64, total_tokens=256, max_n=64, phi="silu", scale=1.0,
                dtype=torch.bfloat16)
    base.update(kw)
    return G.problem(**base)


def test_workspace_sizes_grow_with_problem():
    small = G.fwd_workspace_bytes(_p())
    big = G.fwd_workspace_bytes(_p(total_tokens=1 << 20, max_n=1 << 19))
    assert 256 <= small < big and small % 256 == 0
    assert G.bwd_workspace_bytes(_p(phi="softmax")) >= small


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), 1), (dict(h=0), 1), (dict(m=0), 1), (dict(dh=48), 2), (dict(dh=256), 2),
    (dict(phi=7), 1), (dict(total_tokens=-1), 1), (dict(max_n=1, total_tokens=256), 1),
    (dict(dtype=torch.float16), 1), (dict(scale=float("nan")), 1),
    (dict(total_tokens=1 << 31, max_n=1 << 30), 1),
])
def test_invalid_problems_rejected_on_host(kw, code):
    with pytest.raises(G.GdpaError) as e:
        G.fwd_workspace_bytes(_p(**kw))
    assert e.value.code == code


def test_null_and_misaligned_pointers_rejected_before_launch():
    lib = pkg.load()
    p = _p()
    ws = ctypes.c_void_p(1 << 20)   # never dereferenced: validation fails first
    args = [ctypes.byref(p), 4096, 8192, 4096, 4096, 4096, None, ws, 1 << 30, None]
    bad_null = list(args)
    bad_null[1] = None
    assert lib.gdpa_fwd(*bad_null) == 1
    bad_align = list(args)
    bad_align[3] = 4096 + 8
    assert lib.gdpa_fwd(*bad_align) == 1
    small_ws = list(args)
    small_ws[8] = 16
    assert lib.gdpa_fwd(*small_ws) == 5
    mis_ws = list(args)
    mis_ws[7] = ctypes.c_void_p((1 << 20) + 64)
    assert lib.gdpa_fwd(*mis_ws) == 5
    # softmax backward needs o and lse
    ps = _p(phi="softmax")
    assert lib.gdpa_bwd(ctypes.byref(ps), 4096, 8192, 4096, 4096, None, None, 4096, 4096,
                        4096, 4096, ws, 1 << 30, None) == 1


def test_selftest_rejects_bad_arguments():
    lib = pkg.load()
    lib.gdpa_selftest_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint32,
                                               ctypes.c_void_p]
    assert lib.gdpa_selftest_wait_timeout(None, 256, 10, None) == 1
    assert lib.gdpa_selftest_wait_timeout(1 << 20, 16, 10, None) == 1
    assert lib.gdpa_selftest_wait_timeout(1 << 20, 256, 0, None) == 1


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(ImportError):
        G.load(str(tmp_path / "libgdpa.so"))


def test_weight_gen_rejects_unsupported_shapes_on_host():
    import ctypes
    lib = pkg.load()
    n = ctypes.c_size_t()
    assert lib.gdpa_weight_gen_bwd_workspace_size(100, 1024, 32, ctypes.byref(n)) == 2
    assert lib.gdpa_weight_gen_bwd_workspace_size(897, 1024, 64, ctypes.byref(n)) == 2
    assert lib.gdpa_weight_gen_bwd_workspace_size(100, 1020, 64, ctypes.byref(n)) == 2
    assert lib.gdpa_weight_gen_bwd_workspace_size(100, 1024, 64, ctypes.byref(n)) == 0
    assert n.value >= 256 + 1024 * 64 * 2 + 100 * 64 * 2
    # argument checks come before any CUDA call
    assert lib.gdpa_weight_gen(4, 64, 48, 4096, 4096, 4096, None, None) == 2
    assert lib.gdpa_weight_gen(4, 60, 64, 4096, 4096, 4096, None, None) == 2
    assert lib.gdpa_weight_gen(4, 64, 64, None, 4096, 4096, None, None) == 1
    assert lib.gdpa_weight_gen(4, 64, 64, 4100, 4096, 4096, None, None) == 1


def test_pool_rejects_unsupported_shapes_on_host():
    import ctypes
    lib = pkg.load()
    n = ctypes.c_size_t()
    assert lib.gdpa_pool_workspace_size(4, 2, 128, 16, ctypes.byref(n)) == 2     # dh 128
    assert lib.gdpa_pool_workspace_size(4, 2, 64, 129, ctypes.byref(n)) == 2     # S > 128
    assert lib.gdpa_pool_workspace_size(4097, 2, 64, 16, ctypes.byref(n)) == 2   # B > 4096
    assert lib.gdpa_pool_workspace_size(0, 2, 64, 16, ctypes.byref(n)) == 1
    assert lib.gdpa_pool_workspace_size(4, 3, 64, 16, ctypes.byref(n)) == 0
    assert n.value >= 256 + 16 * 4 * 2


def test_pool_and_window_backward_check_arguments_on_host():
    """Shape limits and workspace sizes of the two backward calls (no launch)."""
    lib = pkg.load()
    G.load()
    n = ctypes.c_size_t()
    assert lib.gdpa_pool_bwd_workspace_size(4, 2, 128, 16, 100, ctypes.byref(n)) == 2
    assert lib.gdpa_pool_bwd_workspace_size(4, 2, 64, 129, 100, ctypes.byref(n)) == 2
    assert lib.gdpa_pool_bwd_workspace_size(4, 2, 64, 16, -1, ctypes.byref(n)) == 1
    assert lib.gdpa_pool_bwd_workspace_size(4, 3, 64, 16, 1000, ctypes.byref(n)) == 0
    # list of h * (T / 128 + B) items and the row sums D [B, h, S]
    assert n.value >= 16 * 3 * (1000 // 128 + 4) + 4 * 4 * 3 * 16
    assert lib.gdpa_window_bwd_workspace_size(4097, 2, 64, 100, ctypes.byref(n)) == 2
    assert lib.gdpa_window_bwd_workspace_size(4, 2, 128, 100, ctypes.byref(n)) == 2
    assert lib.gdpa_window_bwd_workspace_size(4, 2, 64, 1000, ctypes.byref(n)) == 0
    # the list, the fp32 dQ accumulator [T, h, dh] and D [h, T]
    assert n.value >= 1000 * 2 * 64 * 4 + 2 * 1000 * 4
    # argument checks come before any CUDA call: window 0, null offsets
    assert lib.gdpa_window_bwd(4, 2, 64, 100, 50, 0, 1.0, *([4096] * 11), 1 << 20, None) == 1
    assert lib.gdpa_window_bwd(4, 2, 64, 100, 50, 8, 1.0, 4096, None, *([4096] * 9), 1 << 20,
                               None) == 1
    assert lib.gdpa_pool_bwd(4, 2, 64, 129, 100, 50, 1.0, *([4096] * 11), 1 << 20, None) == 2
    assert lib.gdpa_pool_bwd(4, 2, 64, 16, 100, 50, 1.0, 4096, None, *([4096] * 9), 1 << 20,
                             None) == 1


def _declared_arity():
    """Parameter count of every GDPA_API function in include/gdpa.h."""
    src = open(os.path.join(ROOT, "include", "gdpa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"GDPA_API\s+[\w\s\*]+?\b(gdpa_\w+)\s*\(([^)]*)\)", src):
        args = m.group(2).strip()
        out[m.group(1)] = 0 if args in ("", "void") else args.count(",") + 1
    return out


def test_binding_argtypes_match_the_header():
    """Every entry point the binding types has exactly the header's number of
    parameters (a missing one would hand the stream to an untyped argument)."""
    lib = G.load()
    arity = _declared_arity()
    typed = 0
    for name, n in arity.items():
        fn = getattr(lib, name)
        if fn.argtypes is not None:
            assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)
            typed += 1
    assert typed >= 20
