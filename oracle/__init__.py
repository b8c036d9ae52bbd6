"""fp64 CPU oracle for the exact attention forward.  TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and it
imports nothing from the CUDA package: the two meet only through the seeded
inputs that the tests pass to both.

The arithmetic lives in ``attention_ref.c`` (plain C, fp64, POSIX threads over
(batch, head, block of query rows)); this file only marshals arrays.  See
that file's header for the definition it follows and the readings taken
where the pages are silent.  Parity pins: ``tests/test_oracle.py``.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

# element encodings: fp64, fp32, bf16 bit patterns (uint16), FP8 E4M3 codes (uint8)
_IN_KIND = {np.dtype(np.float64): 0, np.dtype(np.float32): 1, np.dtype(np.uint16): 2,
            np.dtype(np.uint8): 3}
_lib = None


def open_library(path: str):
    """Bind a compiled copy of attention_ref.c (the default one, or a test's
    deliberately mutated copy)."""
    lib = ctypes.CDLL(path)
    lib.oracle_attention_fwd_general.restype = ctypes.c_int
    lib.oracle_attention_fwd_general.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
    ]
    lib.oracle_attention_bwd.restype = ctypes.c_int
    lib.oracle_attention_bwd.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
        ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_int,
    ]
    lib.oracle_attention_fwd.restype = ctypes.c_int
    lib.oracle_attention_fwd.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
    ]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = open_library(_build.build())
    return _lib


def num_threads() -> int:
    """Threads the oracle uses: the cores this process may run on."""
    import os
    return max(1, len(os.sched_getaffinity(0)))


def attention_forward(q, k, v, *, causal: bool, scale: float, seqlens=None, rows=None,
                      return_probs: bool = False, threads: int | None = None,
                      causal_bottom_right: bool = False, _lib_override=None):
    """Exact softmax attention in fp64.

    q: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d]; dtype float64, float32, uint16
    (bf16 bit patterns) or uint8 (FP8 E4M3 codes).  seqlens: int [B] key lengths or None.  rows: int
    [B*Hq, R] query rows per (batch, head) or None for all rows.
    causal_bottom_right: with causal, query i sits at position len_b - Nq + i
    (key j visible iff j <= i + len_b - Nq); otherwise causal is top-left.

    Returns (o [B, Hq, R, d], lse [B, Hq, R]) in fp64, plus P [B, Hq, R, Nk]
    when return_probs is set (small cases only).
    """
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    if not (q.dtype == k.dtype == v.dtype) or q.dtype not in _IN_KIND:
        raise TypeError("q, k, v must share one dtype among float64, float32, uint16(bf16), "
                        "uint8(e4m3)")
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if (Bk, dk) != (B, d) or v.shape != k.shape:
        raise ValueError("shape mismatch between q and k/v")
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    sl = None
    if seqlens is not None:
        sl = np.ascontiguousarray(seqlens, dtype=np.int32)
        if sl.shape != (B,) or np.any(sl < 0) or np.any(sl > Nk):
            raise ValueError("seqlens must be int[B] within [0, Nk]")
    if rows is None:
        R = Nq
        rw = None
    else:
        rw = np.ascontiguousarray(rows, dtype=np.int64)
        if rw.ndim != 2 or rw.shape[0] != B * Hq or np.any(rw < 0) or np.any(rw >= Nq):
            raise ValueError("rows must be int[B*Hq, R] within [0, Nq)")
        R = rw.shape[1]
    o = np.empty((B, Hq, R, d), dtype=np.float64)
    lse = np.empty((B, Hq, R), dtype=np.float64)
    p = np.empty((B, Hq, R, Nk), dtype=np.float64) if return_probs else None

    def ptr(a):
        return None if a is None else a.ctypes.data_as(ctypes.c_void_p)

    lib = _lib_override if _lib_override is not None else _load()
    rc = lib.oracle_attention_fwd_general(
        ptr(q), ptr(k), ptr(v), _IN_KIND[q.dtype], B, Hq, Hkv, Nq, Nk, d, float(scale),
        int(bool(causal)), int(bool(causal_bottom_right)), ptr(sl), ptr(rw), R, ptr(o),
        ptr(lse), ptr(p), int(threads or num_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle_attention_fwd failed ({rc})")
    return (o, lse, p) if return_probs else (o, lse)


def attention_backward(q, k, v, dout, *, causal: bool, scale: float, seqlens=None,
                       threads: int | None = None, _lib_override=None):
    """Gradients (dq, dk, dv) in fp64 of sum(dout * O), O = attention_forward.

    q, dout: [B, Hq, N, d]; k, v: [B, Hkv, N, d], one dtype among float64,
    float32 and uint16 (bf16 bit patterns).  dk and dv sum over the query
    heads that share each kv head."""
    q, k, v, dout = (np.ascontiguousarray(x) for x in (q, k, v, dout))
    if not (q.dtype == k.dtype == v.dtype == dout.dtype) or q.dtype not in _IN_KIND:
        raise TypeError("q, k, v, dout must share one dtype among float64, float32, uint16(bf16)")
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape or dout.shape != q.shape:
        raise ValueError("shape mismatch")
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    sl = None
    if seqlens is not None:
        sl = np.ascontiguousarray(seqlens, dtype=np.int32)
        if sl.shape != (B,) or np.any(sl < 0) or np.any(sl > N):
            raise ValueError("seqlens must be int[B] within [0, N]")
    dq = np.empty(q.shape, dtype=np.float64)
    dk = np.empty(k.shape, dtype=np.float64)
    dv = np.empty(k.shape, dtype=np.float64)

    def ptr(a):
        return None if a is None else a.ctypes.data_as(ctypes.c_void_p)

    lib = _lib_override if _lib_override is not None else _load()
    rc = lib.oracle_attention_bwd(ptr(q), ptr(k), ptr(v), ptr(dout), _IN_KIND[q.dtype], B, Hq,
                                  Hkv, N, d, float(scale), int(bool(causal)), ptr(sl), ptr(dq),
                                  ptr(dk), ptr(dv), int(threads or num_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle_attention_bwd failed ({rc})")
    return dq, dk, dv
