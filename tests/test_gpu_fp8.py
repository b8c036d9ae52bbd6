"""FP8 forward (fa_fwd_fp8) vs the fp64 oracle on the same E4M3 codes.

The oracle runs on the codes themselves (it decodes E4M3 exactly) with the
scale multiplied by the Q and K descales; O is linear in V, so its result
times the V descale is the exact attention of the quantised inputs.

Tolerance (the pages give none for FP8; derived from the kernel's
arithmetic).  The scores are exact products of 8-bit values summed in fp32,
and the row sum l adds the fp32 probabilities, so LSE keeps the bf16 path's
2e-3.  The probabilities enter the P.V product as E4M3 codes: the kernel
stores p' = p * 2^c, with p = exp(s - max) and 2 <= c <= 8 (a factor 2^2
plus the lag of at most 2^6 of its reference max).  A normal code is within
a relative 2^-4 of p', and a subnormal one (p' < 2^-6) is within 2^-10
absolute.  With w = p / sum(p), w_max = 1 / sum(p), and the exponential's
own relative error (at most 7.5e-5), each output element of row i obeys

  |O - O_ref| <= dv * sum_j |v_j| (max(2^-4 w_j, 2^-12 w_max) + 7.5e-5 w_j)
                 + 2^-9 |O_ref| + 1e-5

where the sum runs over the keys the row sees (w_j > 0), v_j are V's codes
and 2^-9 |O_ref| is the bf16 rounding of O.  The test requires this of every
element and reports the largest ratio error / bound."""
import numpy as np
import pytest

from exact_io_aware_92_b200 import workloads as wl

pytestmark = pytest.mark.gpu

import oracle  # noqa: E402

LSE_TOL = 2e-3


def _decode(codes):
    import torch
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(
        torch.float64).numpy()


def _bounds(p, v_vals, o_ref, group):
    """Per-element bound for rows whose exact weights are p [B, Hq, R, N]."""
    B, Hq, R, N = p.shape
    out = np.empty_like(o_ref)
    for b in range(B):
        for h in range(Hq):
            w = p[b, h]
            wmax = w.max(axis=1, keepdims=True)
            term = np.where(w > 0, np.maximum(2.0 ** -4 * w, 2.0 ** -12 * wmax) + 7.5e-5 * w, 0.0)
            out[b, h] = term @ np.abs(v_vals[b, h // group])
    return out + 2.0 ** -9 * np.abs(o_ref) + 1e-5


def run_case(B, Hq, Hkv, N, causal, seed, *, seqlens=None, k_scale=1.0, ldvt=None, rows=None):
    import torch
    from exact_io_aware_92_b200 import attention
    d = 128
    inp = wl.draw_fp8(B, Hq, Hkv, N, d, seed, k_scale=k_scale)
    if seqlens is not None:
        inp.seqlens = np.asarray(seqlens, dtype=np.int32)
    scale = 1.0 / np.sqrt(d)
    q = torch.from_numpy(inp.q).cuda()
    k = torch.from_numpy(inp.k).cuda()
    vt = torch.from_numpy(inp.vt(ldvt)).cuda()
    sl = None if inp.seqlens is None else torch.from_numpy(inp.seqlens).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = attention.fwd_fp8(q, k, vt, descale_q=inp.descale_q, descale_k=inp.descale_k,
                               descale_v=inp.descale_v, causal=causal, scale=scale, seqlens=sl,
                               status=status)
    assert attention.check_status(status) == 0
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o))
    # the kernel's scale: fp32(scale) * descale_q * descale_k
    s_eff = float(np.float32(scale)) * inp.descale_q * inp.descale_k
    o_ref, lse_ref, p = oracle.attention_forward(inp.q, inp.k, inp.v, causal=causal, scale=s_eff,
                                                 seqlens=inp.seqlens, rows=rows,
                                                 return_probs=True)
    o_ref = o_ref * inp.descale_v
    if rows is not None:
        o = np.take_along_axis(o.reshape(B * Hq, N, d), rows[:, :, None], axis=1).reshape(
            o_ref.shape)
        lse = np.take_along_axis(lse.reshape(B * Hq, N), rows, axis=1).reshape(lse_ref.shape)
    bound = _bounds(p, _decode(inp.v) * inp.descale_v, o_ref, Hq // Hkv)
    err = np.abs(o - o_ref)
    ratio = float((err / bound).max())
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), fin), "rows without keys must give LSE = -inf"
    lse_err = float(np.abs(lse[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    assert ratio <= 1.0, f"max |dO| / bound = {ratio:.3f} (max |dO| {err.max():.3e})"
    assert lse_err <= LSE_TOL, f"max |dLSE| {lse_err:.3e}"
    return {"max_err": float(err.max()), "max_ratio": ratio,
            "mean_ratio": float((err / bound).mean()), "lse_err": lse_err}


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 128, 129, 300, 513])
def test_fp8_ragged_lengths(N, causal):
    print(run_case(1, 2, 1, N, causal, seed=1600 + N))


def test_fp8_gqa_padding_and_pitch():
    print(run_case(3, 8, 2, 300, True, seed=1700, seqlens=[300, 0, 150], ldvt=352))
    print(run_case(2, 4, 4, 260, False, seed=1701, seqlens=[1, 260]))


def test_fp8_sharpened_scores():
    # K x 8: near one-hot rows, large jumps of the row max between tiles
    print(run_case(1, 4, 1, 700, True, seed=1702, k_scale=8.0))


def test_fp8_full_gqa_workload_sampled_rows():
    w = wl.LLAMA_GQA_FP8
    rows = wl.sample_rows(w, 16)
    print(run_case(w.B, w.Hq, w.Hkv, w.N, w.causal, w.seed, k_scale=w.k_scale, rows=rows))


def test_fp8_kv_beyond_l2_sampled_rows():
    # 134 MB of E4M3 K/V, more than the L2, 32 heads of 16384 keys
    w = wl.Workload("fp8_kv_beyond_l2", 1, 32, 32, 16384, 128, True, seed=2200)
    rows = wl.sample_rows(w, 16)
    print(run_case(1, 32, 32, 16384, True, 2200, k_scale=2.0, rows=rows))
