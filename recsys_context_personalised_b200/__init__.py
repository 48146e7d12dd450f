"""B200-native (sm_100a) GDPA: Generalized Dot-Product Attention.

GDPA is the Kunlun recommendation model's Personalized FFN recast as a
multi-head attention operator: jagged user-history tokens are the queries,
per-sample context-generated weights are the keys and values, and
O = phi(s Q K^T) V with phi in {identity, SiLU, softmax, ReLU, GELU}.  The compute runs in
libgdpa.so (CUDA C++ for sm_100a behind a C ABI, ``include/gdpa.h``);
``gdpa`` is its ctypes binding.
"""
from . import gdpa  # noqa: F401
from .gdpa import (GdpaError, Problem, bwd, bwd_bias, bwd_workspace_bytes, fwd,  # noqa: F401
                   fwd_bias, fwd_workspace_bytes, load, problem, problem_for, workspace,
                   workspace_status)

__all__ = ["gdpa", "GdpaError", "Problem", "fwd", "bwd", "fwd_bias", "bwd_bias",
           "fwd_workspace_bytes",
           "bwd_workspace_bytes", "load", "problem", "problem_for", "workspace",
           "workspace_status"]
