"""Exact, IO-aware attention for B200 (sm_100a): forward (bf16 and FP8),
backward, packed variable-length and split-KV decode.

The computation lives in hand-written CUDA kernels behind the C ABI of
``include/fa.h`` (``libfa_b200.so``); this package holds the ctypes binding
(``attention``), the in-place build (``build``) and the seeded synthetic
inputs (``workloads``).
"""
from . import workloads  # noqa: F401

_API = ("fwd", "bwd", "fwd_fp8", "fwd_varlen", "fwd_decode", "decode_workspace_size", "bwd_workspace_size",
        "check_status", "fwd_hostio", "measure_ex2_rate")
__all__ = list(_API) + ["workloads"]


def __getattr__(name):
    if name in _API:
        from . import attention
        return getattr(attention, name)
    raise AttributeError(name)
