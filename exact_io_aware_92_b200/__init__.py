"""Exact, IO-aware attention forward for B200 (sm_100a).

The computation lives in hand-written CUDA kernels behind the C ABI of
``include/fa.h`` (``libfa_b200.so``); this package holds the ctypes binding
(``attention``), the in-place build (``build``) and the seeded synthetic
inputs (``workloads``).
"""
from . import workloads  # noqa: F401

__all__ = ["fwd", "fwd_varlen", "fwd_decode", "decode_workspace_size", "check_status", "fwd_hostio",
           "workloads"]


def __getattr__(name):
    if name in ("fwd", "fwd_varlen", "fwd_decode", "decode_workspace_size", "check_status", "fwd_hostio"):
        from . import attention
        return getattr(attention, name)
    raise AttributeError(name)
