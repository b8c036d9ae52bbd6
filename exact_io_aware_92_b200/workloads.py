"""Seeded synthetic inputs for the attention kernels.

This module only draws numbers and rounds them to bf16 (or quantises them to
FP8 E4M3 with one scale per tensor); it holds none of the attention
arithmetic.  Both the CUDA path (through the binding) and the CPU
oracle consume what it produces, so neither has to import the other.

Recipe (the same for every workload):
  * ``numpy.random.default_rng(seed)`` (PCG64) draws fp32 ``standard_normal``
    in the order Q, K, V, each of shape ``[B, H, N, d]`` (K and V use the KV
    head count);
  * K is multiplied by ``k_scale`` before rounding (2.0 for the GQA workload,
    an exact power-of-two scaling);
  * every tensor is rounded to bf16 with round-to-nearest-even; the fp32 copy
    that the oracle reads holds exactly those bf16 values;
  * key-padded workloads then draw ``seqlens = rng.integers(lo, hi + 1, B)``
    from the same generator;
  * sampled-row checks draw their query rows from ``default_rng(seed + 100)``
    without replacement, independently per (batch, head);
  * FP8 inputs take the same fp32 draws and quantise each tensor to E4M3
    codes with descale = amax / 448 (round to nearest even, PyTorch's
    float8_e4m3fn cast); V is also laid out transposed, keys contiguous.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    seed: int
    k_scale: float = 1.0
    seqlen_range: tuple[int, int] | None = None  # inclusive [lo, hi] key lengths
    sample_rows: int | None = None  # oracle rows per head for large cases
    nq: int | None = None  # query rows for the decode shape (keys: N); None = N

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


# The five workloads the pages' problem statement is measured on (shapes of
# GPT-2 small, BERT-large with padding, a Llama-style GQA layer and a long
# context), plus the tiny exact case.
TINY = Workload("tiny_b1_h2_n256_d64", 1, 2, 2, 256, 64, False, seed=1)
GPT2 = Workload("gpt2_causal_b8_h12_n1024_d64", 8, 12, 12, 1024, 64, True, seed=2)
BERT = Workload("bert_padded_b16_h16_n512_d64", 16, 16, 16, 512, 64, False, seed=3,
                seqlen_range=(64, 512))
LLAMA_GQA = Workload("llama_gqa_causal_b2_hq32_hkv8_n8192_d128", 2, 32, 8, 8192, 128, True,
                     seed=4, k_scale=2.0, sample_rows=256)
LONG = Workload("long_causal_b1_h16_n32768_d128", 1, 16, 16, 32768, 128, True, seed=5,
                sample_rows=256)

# Decode against a KV cache (wiki note "FlashAttention", common misconceptions:
# one generated token is bound by reading the cache): one new token per
# sequence, the Llama-style GQA heads, caches of 16K-32K tokens.
DECODE = Workload("llama_gqa_decode_b8_hq32_hkv8_nq1_nk32768_d128", 8, 32, 8, 32768, 128, True,
                  seed=6, seqlen_range=(16384, 32768), nq=1)
# Group size 8 (32 query heads on 4 kv heads) with 4 new query rows per
# sequence (speculative or chunked decode): 8 x 4 = 32 query rows per kv head,
# caches of 16K-32K tokens.
DECODE_NQ4 = Workload("gqa8_decode_b8_hq32_hkv4_nq4_nk32768_d128", 8, 32, 4, 32768, 128,
                      True, seed=7, seqlen_range=(16384, 32768), nq=4)

ALL = (TINY, GPT2, BERT, LLAMA_GQA, LONG)
# The GQA workload with FP8 E4M3 inputs (the same draws, quantised).
LLAMA_GQA_FP8 = Workload("llama_gqa_causal_b2_hq32_hkv8_n8192_d128_e4m3", 2, 32, 8, 8192, 128,
                         True, seed=4, k_scale=2.0, sample_rows=32)

BY_NAME = {w.name: w for w in ALL + (DECODE, DECODE_NQ4, LLAMA_GQA_FP8)}


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest, ties to even.

    Inputs here are finite normal draws, so no NaN handling is needed; a NaN
    or an infinity is rejected rather than silently re-encoded."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.size <= (1 << 20):
        if not np.all(np.isfinite(x)):
            raise ValueError("round_to_bf16_bits: non-finite input")
        # Finite fp32 bit patterns are <= 0xFF7FFFFF, so adding at most
        # 0x8000 cannot overflow 32 bits.
        u = x.view(np.uint32)
        r = u + np.uint32(0x7FFF)
        r += (u >> np.uint32(16)) & np.uint32(1)
        r >>= np.uint32(16)
        return r.astype(np.uint16)
    # Large tensors: the same rounding (fp32 -> bf16 is round-to-nearest-even
    # in PyTorch too; tests/test_workloads.py checks the two agree), multithreaded.
    import torch
    t = torch.from_numpy(x)
    if not bool(torch.isfinite(t).all()):
        raise ValueError("round_to_bf16_bits: non-finite input")
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> the fp32 values they encode (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class Inputs:
    """One seeded draw.  ``*_bits`` are the bf16 tensors the kernels read;
    ``*_f32`` hold exactly the same values in fp32 for the oracle and for the
    fp32 check mode."""
    q_bits: np.ndarray
    k_bits: np.ndarray
    v_bits: np.ndarray
    seqlens: np.ndarray | None  # int32 [B] or None

    @property
    def q_f32(self) -> np.ndarray:
        return bf16_bits_to_f32(self.q_bits)

    @property
    def k_f32(self) -> np.ndarray:
        return bf16_bits_to_f32(self.k_bits)

    @property
    def v_f32(self) -> np.ndarray:
        return bf16_bits_to_f32(self.v_bits)


def draw(B: int, Hq: int, Hkv: int, N: int, d: int, seed: int, *, k_scale: float = 1.0,
         seqlen_range: tuple[int, int] | None = None, nq: int | None = None) -> Inputs:
    """Q has nq rows (default N: self-attention); K and V have N rows."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, N if nq is None else nq, d), dtype=np.float32)
    k = rng.standard_normal((B, Hkv, N, d), dtype=np.float32)
    v = rng.standard_normal((B, Hkv, N, d), dtype=np.float32)
    if k_scale != 1.0:
        k *= np.float32(k_scale)
    seqlens = None
    if seqlen_range is not None:
        lo, hi = seqlen_range
        seqlens = rng.integers(lo, hi + 1, B).astype(np.int32)
    return Inputs(round_to_bf16_bits(q), round_to_bf16_bits(k), round_to_bf16_bits(v), seqlens)


def pack(x: np.ndarray, lengths) -> np.ndarray:
    """[B, H, N, d] -> the packed layout [sum(lengths), H, d] (rows of each
    sequence below its length, sequences back to back)."""
    return np.ascontiguousarray(np.concatenate(
        [np.transpose(x[b, :, :int(L), :], (1, 0, 2)) for b, L in enumerate(lengths)], axis=0))


def cu_seqlens(lengths) -> np.ndarray:
    """Token offsets [B+1] of sequences stored back to back."""
    return np.concatenate([[0], np.cumsum(np.asarray(lengths, dtype=np.int64))]).astype(np.int32)


def draw_workload(w: Workload) -> Inputs:
    return draw(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, k_scale=w.k_scale,
                seqlen_range=w.seqlen_range, nq=w.nq)


def sample_rows(w: Workload, rows_per_head: int | None = None) -> np.ndarray:
    """Query rows to check for a large workload: int64 [B*Hq, R], sorted per
    (batch, head), drawn without replacement from ``default_rng(seed + 100)``."""
    r = rows_per_head or w.sample_rows or w.N
    rng = np.random.default_rng(w.seed + 100)
    out = np.empty((w.B * w.Hq, r), dtype=np.int64)
    for bh in range(w.B * w.Hq):
        out[bh] = np.sort(rng.choice(w.N, size=r, replace=False))
    return out


def flops(w: Workload, seqlens: np.ndarray | None = None) -> float:
    """Attention forward FLOPs as the metric counts them: 4*B*Hq*N^2*d,
    halved for causal; with key padding 4*Hq*d*N*sum(len_b)."""
    if seqlens is not None:
        return 4.0 * w.Hq * w.d * w.N * float(np.sum(seqlens))
    f = 4.0 * w.B * w.Hq * w.N * w.N * w.d
    return f / 2 if w.causal else f


# ---------------------------------------------------------------------------
# FP8 E4M3 inputs
# ---------------------------------------------------------------------------
E4M3_MAX = 448.0


def quantize_e4m3(x: np.ndarray) -> tuple[np.ndarray, float]:
    """fp32 -> (E4M3 codes as uint8, descale): descale = amax / 448 in fp32,
    codes = x / descale rounded to nearest even by PyTorch's float8_e4m3fn
    cast (clamped to +-448 first), so code * descale approximates x."""
    import torch
    x = np.ascontiguousarray(x, dtype=np.float32)
    amax = float(np.max(np.abs(x))) if x.size else 0.0
    descale = np.float32(amax / E4M3_MAX) if amax > 0 else np.float32(1.0)
    t = (torch.from_numpy(x) / torch.tensor(descale, dtype=torch.float32))
    t = t.clamp(-E4M3_MAX, E4M3_MAX)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy(), float(descale)


def e4m3_transpose(v_codes: np.ndarray, ldvt: int | None = None) -> np.ndarray:
    """[B, H, N, d] codes -> [B, H, d, ldvt] (keys contiguous), zero padded
    past N; ldvt defaults to N rounded up to 16."""
    B, H, N, d = v_codes.shape
    ld = ldvt if ldvt is not None else (N + 15) // 16 * 16
    if ld < N:
        raise ValueError("ldvt must be >= N")
    out = np.zeros((B, H, d, ld), dtype=np.uint8)
    out[..., :N] = np.swapaxes(v_codes, 2, 3)
    return out


@dataclasses.dataclass
class Fp8Inputs:
    """One seeded draw quantised to E4M3: ``q``, ``k``, ``v`` are codes
    [B, H, N, d]; element value = code * descale of its tensor."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    descale_q: float
    descale_k: float
    descale_v: float
    seqlens: np.ndarray | None

    def vt(self, ldvt: int | None = None) -> np.ndarray:
        return e4m3_transpose(self.v, ldvt)


def draw_fp8(B: int, Hq: int, Hkv: int, N: int, d: int, seed: int, *, k_scale: float = 1.0,
             seqlen_range: tuple[int, int] | None = None) -> Fp8Inputs:
    """The fp32 draws of ``draw`` (same seed, same order), each tensor
    quantised to E4M3 with its own scale."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, N, d), dtype=np.float32)
    k = rng.standard_normal((B, Hkv, N, d), dtype=np.float32)
    v = rng.standard_normal((B, Hkv, N, d), dtype=np.float32)
    if k_scale != 1.0:
        k *= np.float32(k_scale)
    seqlens = None
    if seqlen_range is not None:
        lo, hi = seqlen_range
        seqlens = rng.integers(lo, hi + 1, B).astype(np.int32)
    (qc, dq), (kc, dk), (vc, dv) = quantize_e4m3(q), quantize_e4m3(k), quantize_e4m3(v)
    return Fp8Inputs(qc, kc, vc, dq, dk, dv, seqlens)


def draw_fp8_workload(w: Workload) -> Fp8Inputs:
    return draw_fp8(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, k_scale=w.k_scale,
                    seqlen_range=w.seqlen_range)
