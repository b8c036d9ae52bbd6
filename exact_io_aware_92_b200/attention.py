"""Python entry points over the C ABI.  Argument marshalling only: every step
of the attention runs in the CUDA kernels of libfa_b200.so.

PyTorch provides device memory and the current stream; nothing here computes.
"""
from __future__ import annotations

import ctypes
import math

import torch

from . import _lib


def _stream_handle(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check_qkv(q, k, v, dtype):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        if t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous [B, H, N, d] tensor")
    B, Hq, N, d = q.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[2] != N or k.shape[3] != d:
        raise ValueError("k and v must be [B, Hkv, N, d] matching q")
    return B, Hq, k.shape[1], N, d


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool = False,
        scale: float | None = None, seqlens: torch.Tensor | None = None,
        out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
        status: torch.Tensor | None = None):
    """Exact attention forward.  q: [B, Hq, N, d], k, v: [B, Hkv, N, d], all
    bf16 (tensor cores) or all fp32 (check mode), contiguous, on one CUDA
    device.  seqlens: int32 [B] key lengths on the same device, or None.
    Returns (o, lse): o like q, lse fp32 [B, Hq, N].  Runs on the current
    stream; `status` (int32 [1] on the device) receives in-kernel time-outs."""
    if q.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("q, k, v must be bf16 or fp32")
    B, Hq, Hkv, N, d = _check_qkv(q, k, v, q.dtype)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    sl_ptr = None
    if seqlens is not None:
        if seqlens.dtype != torch.int32 or seqlens.device != q.device or seqlens.numel() != B:
            raise ValueError("seqlens must be int32 [B] on q's device")
        sl_ptr = seqlens.data_ptr()
    dtype = _lib.FA_DTYPE_BF16 if q.dtype == torch.bfloat16 else _lib.FA_DTYPE_F32
    rc = _lib.load().fa_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                               lse.data_ptr(), B, Hq, Hkv, N, d, scale, int(bool(causal)), sl_ptr,
                               dtype, _stream_handle(q.device),
                               None if status is None else status.data_ptr())
    _lib.check(rc, "fa_fwd_ex")
    return out, lse


def _codes(t: torch.Tensor, name: str) -> torch.Tensor:
    if not t.is_cuda or t.dtype not in (torch.uint8, torch.float8_e4m3fn) or t.dim() != 4 \
            or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous 4-D uint8 / float8_e4m3fn CUDA tensor")
    return t


def fwd_fp8(q: torch.Tensor, k: torch.Tensor, vt: torch.Tensor, *, descale_q: float,
            descale_k: float, descale_v: float, causal: bool = False,
            scale: float | None = None, seqlens: torch.Tensor | None = None,
            out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
            status: torch.Tensor | None = None):
    """Attention forward on FP8 E4M3 codes with per-tensor descales (value =
    code * descale).  q: [B, Hq, N, 128], k: [B, Hkv, N, 128], vt: V
    transposed [B, Hkv, 128, ldvt] (ldvt >= N, a multiple of 16); uint8 or
    float8_e4m3fn, contiguous.  Returns (o bf16 [B, Hq, N, 128], lse fp32
    [B, Hq, N])."""
    q, k, vt = _codes(q, "q"), _codes(k, "k"), _codes(vt, "vt")
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or vt.shape[:3] != (B, Hkv, d):
        raise ValueError("k must be [B, Hkv, N, d] and vt [B, Hkv, d, ldvt]")
    ldvt = vt.shape[3]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    sl_ptr = None
    if seqlens is not None:
        if seqlens.dtype != torch.int32 or seqlens.device != q.device or seqlens.numel() != B:
            raise ValueError("seqlens must be int32 [B] on q's device")
        sl_ptr = seqlens.data_ptr()
    rc = _lib.load().fa_fwd_fp8(q.data_ptr(), k.data_ptr(), vt.data_ptr(), out.data_ptr(),
                                lse.data_ptr(), B, Hq, Hkv, N, ldvt, d, scale, float(descale_q),
                                float(descale_k), float(descale_v), int(bool(causal)), sl_ptr,
                                _stream_handle(q.device),
                                None if status is None else status.data_ptr())
    _lib.check(rc, "fa_fwd_fp8")
    return out, lse


def bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
        dout: torch.Tensor, lse: torch.Tensor, *, causal: bool = False,
        scale: float | None = None, seqlens: torch.Tensor | None = None,
        workspace: torch.Tensor | None = None, status: torch.Tensor | None = None):
    """Attention backward by recomputation.  q, o, dout: [B, Hq, N, d];
    k, v: [B, Hkv, N, d] (bf16, contiguous); lse: fp32 [B, Hq, N] from fwd
    with the same arguments.  Returns (dq, dk, dv) in bf16."""
    B, Hq, Hkv, N, d = _check_qkv(q, k, v, torch.bfloat16)
    for name, t in (("o", o), ("dout", dout)):
        if t.shape != q.shape or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 tensor shaped like q")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    if workspace is None:
        workspace = torch.empty(bwd_workspace_size(B, Hq, N), dtype=torch.uint8, device=q.device)
    sl_ptr = None
    if seqlens is not None:
        if seqlens.dtype != torch.int32 or seqlens.device != q.device or seqlens.numel() != B:
            raise ValueError("seqlens must be int32 [B] on q's device")
        sl_ptr = seqlens.data_ptr()
    rc = _lib.load().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                            dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                            dv.data_ptr(), B, Hq, Hkv, N, d, scale, int(bool(causal)), sl_ptr,
                            workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                            _stream_handle(q.device),
                            None if status is None else status.data_ptr())
    _lib.check(rc, "fa_bwd")
    return dq, dk, dv


def fwd_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
               max_seqlen: int, *, causal: bool = False, scale: float | None = None,
               out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
               status: torch.Tensor | None = None):
    """Packed variable-length forward.  q: [total, Hq, d], k, v: [total, Hkv, d]
    bf16 contiguous; cu_seqlens: int32 [B+1] token offsets on the device;
    max_seqlen >= every sequence length.  Returns (o [total, Hq, d],
    lse [Hq, total])."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 3 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 [total, H, d] CUDA tensor")
    total, Hq, d = q.shape
    if k.shape != v.shape or k.shape[0] != total or k.shape[2] != d:
        raise ValueError("k and v must be [total, Hkv, d] matching q")
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.device != q.device or cu_seqlens.dim() != 1:
        raise ValueError("cu_seqlens must be int32 [B+1] on q's device")
    B = cu_seqlens.numel() - 1
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hq, total), dtype=torch.float32, device=q.device)
    rc = _lib.load().fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                   lse.data_ptr(), cu_seqlens.data_ptr(), B, Hq, k.shape[1],
                                   total, int(max_seqlen), d, scale, int(bool(causal)),
                                   _stream_handle(q.device),
                                   None if status is None else status.data_ptr())
    _lib.check(rc, "fa_fwd_varlen")
    return out, lse


def bwd_workspace_size(B: int, Hq: int, N: int) -> int:
    """Bytes of device workspace bwd needs (per-row D and LSE*log2(e))."""
    return int(_lib.load().fa_bwd_workspace_size(B, Hq, N))


def decode_workspace_size(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int,
                          num_splits: int = 0) -> int:
    """Bytes of device workspace fwd_decode needs for this shape."""
    return int(_lib.load().fa_decode_workspace_size(B, Hq, Hkv, Nq, Nk, d, num_splits))


def fwd_decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool = False,
               scale: float | None = None, seqlens: torch.Tensor | None = None,
               num_splits: int = 0, workspace: torch.Tensor | None = None,
               out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
               status: torch.Tensor | None = None):
    """Split-KV decode forward.  q: [B, Hq, Nq, d], k, v: [B, Hkv, Nk, d]
    (the cache), bf16, contiguous, one CUDA device.  seqlens: int32 [B]
    valid cache lengths or None.  Causal queries sit at the end of their
    sequence.  workspace: a byte tensor of at least decode_workspace_size()
    bytes (allocated here when None).  Returns (o, lse)."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 4 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 [B, H, N, d] CUDA tensor")
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if (Bk, dk) != (B, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, Nk, d] matching q")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    need = decode_workspace_size(B, Hq, Hkv, Nq, Nk, d, num_splits)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    sl_ptr = None
    if seqlens is not None:
        if seqlens.dtype != torch.int32 or seqlens.device != q.device or seqlens.numel() != B:
            raise ValueError("seqlens must be int32 [B] on q's device")
        sl_ptr = seqlens.data_ptr()
    rc = _lib.load().fa_fwd_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                   lse.data_ptr(), B, Hq, Hkv, Nq, Nk, d, scale,
                                   int(bool(causal)), sl_ptr, int(num_splits),
                                   workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                   _stream_handle(q.device),
                                   None if status is None else status.data_ptr())
    _lib.check(rc, "fa_fwd_decode")
    return out, lse


def check_status(status: torch.Tensor | None = None, device: torch.device | None = None) -> int:
    """Synchronise the current stream and return the status word (0 = ok)."""
    dev = status.device if status is not None else (device or torch.device("cuda"))
    return _lib.load().fa_check_status(None if status is None else status.data_ptr(),
                                       _stream_handle(dev))


def measure_ex2_rate(device: torch.device | None = None) -> float:
    """Calibration: exponentials (ex2.approx.ftz.f32) per SM clock on the
    current device, the median over SMs (fa_measure_ex2_rate)."""
    dev = device or torch.device("cuda")
    out = ctypes.c_float(0.0)
    _lib.check(_lib.load().fa_measure_ex2_rate(ctypes.byref(out), _stream_handle(dev)),
               "fa_measure_ex2_rate")
    return float(out.value)


def fwd_hostio(q_h, k_h, v_h, o_h, lse_h, q_d, k_d, v_d, o_d, lse_d, *, causal: bool,
               scale: float, seqlens_h=None, seqlens_d=None, wait: bool = True) -> None:
    """End-to-end call on host tensors (pinned for asynchronous copies):
    host->device copies, the forward, device->host copies, then a wait.
    wait=False (fa_fwd_hostio_async): return once queued on the current
    stream; consecutive such calls on the same buffers overlap (see fa.h)."""
    B, Hq, N, d = q_h.shape
    Hkv = k_h.shape[1]
    lib = _lib.load()
    rc = (lib.fa_fwd_hostio if wait else lib.fa_fwd_hostio_async)(
        q_h.data_ptr(), k_h.data_ptr(), v_h.data_ptr(), o_h.data_ptr(), lse_h.data_ptr(),
        None if seqlens_h is None else seqlens_h.data_ptr(), q_d.data_ptr(), k_d.data_ptr(),
        v_d.data_ptr(), o_d.data_ptr(), lse_d.data_ptr(),
        None if seqlens_d is None else seqlens_d.data_ptr(), B, Hq, Hkv, N, d, float(scale),
        int(bool(causal)), _stream_handle(q_d.device))
    _lib.check(rc, "fa_fwd_hostio" if wait else "fa_fwd_hostio_async")
