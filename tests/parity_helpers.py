"""Shared pieces of the GPU parity tests: upload seeded inputs, run the CUDA
path through the C ABI binding, run the oracle on the same values, compare.

Tolerances (fixed by the problem statement):
  bf16 path : max |O - O_ref| <= 1.5e-2 and max |LSE - LSE_ref| <= 2e-3
  fp32 path : both <= 1e-5
"""
from __future__ import annotations

import numpy as np

import oracle
from exact_io_aware_92_b200 import workloads as wl

O_TOL_BF16 = 1.5e-2
LSE_TOL_BF16 = 2e-3
TOL_F32 = 1e-5


def to_device_bf16(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).cuda()


def to_device_f32(x: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def run_bf16(inp: wl.Inputs, *, causal: bool, scale: float):
    """CUDA path on bf16 inputs -> (O as fp64 numpy, LSE fp64 numpy)."""
    import torch
    from exact_io_aware_92_b200 import attention
    q, k, v = (to_device_bf16(x) for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    sl = None if inp.seqlens is None else torch.from_numpy(inp.seqlens).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = attention.fwd(q, k, v, causal=causal, scale=scale, seqlens=sl, status=status)
    rc = attention.check_status(status)
    assert rc == 0, f"kernel status {rc}"
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def run_f32(inp: wl.Inputs, *, causal: bool, scale: float):
    import torch
    from exact_io_aware_92_b200 import attention
    q, k, v = (to_device_f32(x) for x in (inp.q_f32, inp.k_f32, inp.v_f32))
    sl = None if inp.seqlens is None else torch.from_numpy(inp.seqlens).cuda()
    o, lse = attention.fwd(q, k, v, causal=causal, scale=scale, seqlens=sl)
    torch.cuda.synchronize()
    return o.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def reference(inp: wl.Inputs, *, causal: bool, scale: float, rows=None, return_probs=False):
    """Oracle on exactly the bf16 values the kernel read (fp32-rounded scale,
    as the kernel receives it)."""
    return oracle.attention_forward(inp.q_bits, inp.k_bits, inp.v_bits, causal=causal,
                                    scale=float(np.float32(scale)), seqlens=inp.seqlens,
                                    rows=rows, return_probs=return_probs)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def gather_rows(o, lse, rows):
    """Pick per-(b, h) rows out of full [B, H, N, ...] outputs."""
    B, H = o.shape[:2]
    og = np.stack([o[bh // H, bh % H, rows[bh]] for bh in range(B * H)]).reshape(
        B, H, rows.shape[1], o.shape[-1])
    lg = np.stack([lse[bh // H, bh % H, rows[bh]] for bh in range(B * H)]).reshape(
        B, H, rows.shape[1])
    return og, lg


# Constants of the per-element bound on the bf16 forward's O (derived_o_bound).
U_ACC = 2.0 ** -23    # fp32 accumulation, allowing truncating adds in the tensor cores
EPS_EXP = 7.5e-5      # relative error of the exponentials (the FMA-pipe polynomial's)
U_P = 2.0 ** -8       # bf16 unit roundoff (8 significant bits): each probability, each dS
ABS_SLACK = 1e-6      # absolute slack for the last fp32 roundings


def derived_o_bound(inp: wl.Inputs, p: np.ndarray, o_ref: np.ndarray, scale: float) -> np.ndarray:
    """Largest |O_gpu - O_ref| a correct bf16 kernel can produce, per element.

    The result equals the exact attention up to floating-point rounding (wiki
    note "FlashAttention", section "what it is"), so the bound adds up the
    roundings the kernel's arithmetic makes, for row i and column c with the
    oracle's exact weights w_ij and A_ic = sum_j w_ij |v_jc|:
      - each probability enters P.V as bf16:               U_P * A_ic
      - each exponential's relative error (numerator and
        row sum, at most EPS_EXP each):                    2 EPS_EXP * A_ic
      - the fp32 scores: |ds_ij| <= d U_ACC sum_k |q_ik k_jk|, times the
        scale, perturbs every weight's exponent; a shift common to the row
        cancels, so weights move by at most 2 Delta_i:     2 Delta_i * A_ic
      - fp32 sums over the n_i visible keys (P.V, row sum), the O rescales
        and the final 1/l:                                 (2 n_i + 8) U_ACC * A_ic
      - then O is rounded to bf16: half an ulp of |O_ref| + E.
    p: the oracle's weights [B, Hq, N, Nk] for every row of inp."""
    q = wl.bf16_bits_to_f32(inp.q_bits).astype(np.float64)
    k = wl.bf16_bits_to_f32(inp.k_bits).astype(np.float64)
    v = wl.bf16_bits_to_f32(inp.v_bits).astype(np.float64)
    B, Hq, N, d = q.shape
    group = Hq // k.shape[1]
    out = np.empty_like(o_ref)
    for b in range(B):
        for h in range(Hq):
            w = p[b, h]
            a = w @ np.abs(v[b, h // group])                       # A_ic
            n = (w > 0).sum(axis=1, keepdims=True)                 # visible keys
            smax = (np.abs(q[b, h]) @ np.abs(k[b, h // group]).T).max(axis=1, keepdims=True)
            delta = abs(scale) * d * U_ACC * smax                  # Delta_i
            e = (U_P + 2 * EPS_EXP + 2 * delta + (2 * n + 8) * U_ACC) * a + ABS_SLACK
            out[b, h] = e + 0.5 * bf16_ulp(np.abs(o_ref[b, h]) + e)
    return out


def compare(o, lse, o_ref, lse_ref, *, o_tol, lse_tol, what="", o_bound=None,
            max_over_tol_frac=1e-4):
    """Element-by-element check.  Rows with no visible key must be O = 0 and
    LSE = -inf exactly on both sides.

    o_bound (stress inputs outside the stated workloads only): where |O_ref|
    >= 4, half a bf16 ulp (1/64) exceeds o_tol, so no bf16 output can be held
    to it.  With o_bound given (derived_o_bound), o_tol stays the floor: an
    element beyond it must lie within its own derived bound, and at most
    max_over_tol_frac of the elements may lie beyond o_tol.  Returns
    (max |dO|, max |dLSE|, elements beyond o_tol)."""
    dead = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), dead), f"{what}: -inf LSE rows differ"
    assert np.all(o[dead] == 0.0), f"{what}: fully masked rows must be 0"
    assert np.all(np.isfinite(o)), f"{what}: non-finite O"
    live = ~dead
    err_o = np.abs(o - o_ref)
    err_l = np.abs(lse[live] - lse_ref[live]) if np.any(live) else np.zeros(1)
    max_o = float(err_o.max()) if err_o.size else 0.0
    max_l = float(err_l.max()) if err_l.size else 0.0
    assert max_l <= lse_tol, f"{what}: max|dLSE| = {max_l:.3e} > {lse_tol}"
    over = err_o > o_tol
    n_over = int(over.sum())
    if o_bound is not None and n_over:
        beyond = over & (err_o > o_bound)
        if np.any(beyond):
            idx = np.unravel_index(np.argmax(np.where(beyond, err_o / o_bound, 0.0)), err_o.shape)
            raise AssertionError(
                f"{what}: |dO| = {err_o[idx]:.3e} beyond its derived bound {o_bound[idx]:.3e} "
                f"at {idx}: gpu {o[idx]!r} ref {o_ref[idx]!r}")
        limit = max_over_tol_frac * err_o.size
        assert n_over <= limit, (f"{what}: {n_over} elements beyond {o_tol} (at most "
                                 f"{limit:.0f} allowed)")
        return max_o, max_l, n_over
    if max_o > o_tol:
        idx = np.unravel_index(np.argmax(err_o), err_o.shape)
        ulps = err_o[idx] / bf16_ulp(o_ref[idx])
        raise AssertionError(
            f"{what}: max|dO| = {max_o:.3e} > {o_tol} at {idx}: gpu {o[idx]!r} ref "
            f"{o_ref[idx]!r} ({ulps:.2f} bf16 ulps of the reference)")
    return max_o, max_l, n_over


def derived_grad_bounds(inp: wl.Inputs, dout_bits: np.ndarray, p: np.ndarray, o_ref: np.ndarray,
                        o_bound: np.ndarray, grads_ref, scale: float):
    """Largest |g_gpu - g_ref| a correct backward can produce, per element of
    dQ, dK and dV, from the roundings its arithmetic makes (the pages give
    no tolerance for gradients; P2's statement that the result equals the
    exact attention up to rounding is applied to the gradient of that
    attention).  The backward rebuilds P = exp(scale S - LSE) from the
    forward's LSE, forms D_i = sum_c dO_ic O_ic from the forward's bf16 O,
    dP = dO V^T and dS = P (dP - D), and feeds bf16 P (for dV) and bf16 dS
    (for dK, dQ) to the tensor cores.  With the oracle's exact P, O, dP, D
    and dS:
      - P in fp32 has relative error eps_P = EPS_EXP + Delta_ij + dLSE_i,
        where Delta_ij = scale d U_ACC sum_k |q_ik k_jk| (fp32 scores) and
        dLSE_i (the forward's LSE) = EPS_EXP + 2 max_j Delta_ij + (n_i+8) U_ACC;
      - dP_ij errs by d U_ACC sum_c |dO_ic v_jc|, D_i by sum_c |dO_ic| dO_bound_ic
        (the forward's O bound) plus d U_ACC sum_c |dO_ic O_ic|;
      - so |ddS_ij| <= P eps_P |dP - D| + P (ddP + dD), then bf16 adds U_P |dS|;
      - dV_j = sum_i bf16(P_ij) dO_i errs by sum_i P_ij (U_P + eps_P) |dO_i|;
        dK_j = scale sum_i dS_ij q_i and dQ_i = scale sum_j dS_ij k_j err by
        scale sum |ddS| |q| (|k|);
      - fp32 sums over n terms add (n + 8) U_ACC times the sum of |terms|, and
        the bf16 result adds half an ulp of |g_ref| + E.
    dK and dV sum these over the query heads that share a kv head.
    Returns (bound_dq, bound_dk, bound_dv)."""
    q = wl.bf16_bits_to_f32(inp.q_bits).astype(np.float64)
    k = wl.bf16_bits_to_f32(inp.k_bits).astype(np.float64)
    v = wl.bf16_bits_to_f32(inp.v_bits).astype(np.float64)
    do = wl.bf16_bits_to_f32(dout_bits).astype(np.float64)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    eq = np.zeros_like(q)
    ek = np.zeros_like(k)
    ev = np.zeros_like(v)
    sk = np.zeros_like(k)   # sum of |terms| of dK, for the accumulation term
    sv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            P = p[b, h]
            Q, K, V, dO = q[b, h], k[b, g], v[b, g], do[b, h]
            vis = P > 0
            n = vis.sum(axis=1)
            dP = dO @ V.T
            D = (dO * o_ref[b, h]).sum(axis=1)
            dS = P * (dP - D[:, None])
            delta = abs(scale) * d * U_ACC * (np.abs(Q) @ np.abs(K).T)
            dmax = np.where(vis, delta, 0.0).max(axis=1) if N else np.zeros(0)
            dlse = EPS_EXP + 2 * dmax + (n + 8) * U_ACC
            eps_p = EPS_EXP + delta + dlse[:, None] + 1e-6
            ddp = d * U_ACC * (np.abs(dO) @ np.abs(V).T)
            dd = (np.abs(dO) * o_bound[b, h]).sum(axis=1) + d * U_ACC * (
                np.abs(dO) * np.abs(o_ref[b, h])).sum(axis=1)
            dds = P * eps_p * np.abs(dP - D[:, None]) + P * (ddp + dd[:, None])
            dds = dds + U_P * (np.abs(dS) + dds)
            ev[b, g] += (P * (U_P + eps_p)).T @ np.abs(dO)
            sv[b, g] += P.T @ np.abs(dO)
            ek[b, g] += abs(scale) * (dds.T @ np.abs(Q))
            sk[b, g] += abs(scale) * (np.abs(dS).T @ np.abs(Q))
            eq[b, h] = abs(scale) * (dds @ np.abs(K)) + (N + 8) * U_ACC * abs(scale) * (
                np.abs(dS) @ np.abs(K))
    ek += (N * G + 8) * U_ACC * sk
    ev += (N * G + 8) * U_ACC * sv
    out = []
    for e, r in zip((eq, ek, ev), grads_ref):
        e = e + ABS_SLACK
        out.append(e + 0.5 * bf16_ulp(np.abs(r) + e))
    return tuple(out)
