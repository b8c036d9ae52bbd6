"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics.

Each pin takes an ``fwd`` callable with the signature of
``oracle.attention_forward`` and raises AssertionError when that
implementation contradicts the fact.  ``tests/test_oracle.py`` runs every pin
against the oracle; ``tests/test_oracle_mutants.py`` runs them against copies
of the oracle with planted mistakes and requires each copy to fail at least
one pin.

What is computed comes from the wiki note "FlashAttention" (section "what it
is": O = softmax(QK^T/sqrt(d))V, P rows are a softmax over each row of S,
masks and heads handled per tile, enable_gqa in the SDPA call).
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "closed_form_cases.json")


def _rng_inputs(seed, B, Hq, Hkv, N, d, scale_k=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, N, d))
    k = rng.standard_normal((B, Hkv, N, d)) * scale_k
    v = rng.standard_normal((B, Hkv, N, d))
    return q, k, v


def pin_golden(fwd):
    """Hand-derived closed-form cases (tests/golden/closed_form_cases.json)."""
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q = np.array(c["q"], dtype=np.float64)
        k = np.array(c["k"], dtype=np.float64)
        v = np.array(c["v"], dtype=np.float64)
        sl = None if c["seqlens"] is None else np.array(c["seqlens"], dtype=np.int32)
        o, lse = fwd(q, k, v, causal=c["causal"], scale=c["scale"], seqlens=sl)
        np.testing.assert_allclose(o, np.array(c["o"], dtype=np.float64), rtol=0, atol=1e-12,
                                   err_msg=c["name"])
        np.testing.assert_allclose(lse, np.array(c["lse"], dtype=np.float64), rtol=0, atol=1e-12,
                                   err_msg=c["name"])


def pin_probs_are_a_row_softmax(fwd):
    """Each row of P is a probability vector over the visible keys: entries
    >= 0, masked entries exactly 0, row sum 1 (the softmax normaliser)."""
    B, Hq, Hkv, N, d = 2, 4, 2, 37, 8
    q, k, v = _rng_inputs(11, B, Hq, Hkv, N, d, 2.0)
    sl = np.array([37, 20], dtype=np.int32)
    for causal in (False, True):
        o, lse, p = fwd(q, k, v, causal=causal, scale=0.3, seqlens=sl, return_probs=True)
        assert np.all(p >= 0)
        np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)
        i = np.arange(N)[:, None]
        j = np.arange(N)[None, :]
        for b in range(B):
            masked = np.broadcast_to(j >= sl[b], (N, N))
            if causal:
                masked = masked | (j > i)
            assert np.all(p[b][:, masked] == 0.0)
            assert np.all(p[b][:, ~masked] > 0.0)
        # O is that P applied to the shared kv head's V rows
        g = np.arange(Hq) // (Hq // Hkv)
        np.testing.assert_allclose(o, np.einsum("bhij,bhjc->bhic", p, v[:, g]), rtol=0, atol=1e-12)


def pin_constant_v(fwd):
    """V constant along the key axis -> O equals that constant, whatever Q, K."""
    B, Hq, Hkv, N, d = 2, 6, 3, 29, 5
    q, k, _ = _rng_inputs(12, B, Hq, Hkv, N, d, 3.0)
    c = np.random.default_rng(13).standard_normal((B, Hkv, 1, d))
    v = np.broadcast_to(c, (B, Hkv, N, d)).copy()
    g = np.arange(Hq) // (Hq // Hkv)
    for causal in (False, True):
        o, _ = fwd(q, k, v, causal=causal, scale=0.7, seqlens=np.array([29, 3], np.int32))
        np.testing.assert_allclose(o, np.broadcast_to(c[:, g], o.shape), rtol=0, atol=1e-13)


def pin_single_visible_key(fwd):
    """len_b = 1 leaves key 0 alone: P = 1 on it, O_i = V_0 and
    LSE_i = scale * q_i . k_0 (a single-term log-sum-exp)."""
    B, Hq, Hkv, N, d = 2, 2, 1, 9, 4
    q, k, v = _rng_inputs(14, B, Hq, Hkv, N, d)
    scale = 0.45
    o, lse = fwd(q, k, v, causal=False, scale=scale, seqlens=np.ones(B, np.int32))
    for b in range(B):
        for h in range(Hq):
            np.testing.assert_array_equal(o[b, h], np.broadcast_to(v[b, 0, 0], (N, d)))
            s0 = np.array([scale * math.fsum(q[b, h, i] * k[b, 0, 0]) for i in range(N)])
            np.testing.assert_allclose(lse[b, h], s0, rtol=0, atol=1e-13)


def pin_causal_first_row(fwd):
    """Causal row 0 sees only key 0: O_0 = V_0 exactly, LSE_0 = scale*q_0.k_0."""
    B, Hq, Hkv, N, d = 1, 3, 3, 17, 6
    q, k, v = _rng_inputs(15, B, Hq, Hkv, N, d)
    o, lse = fwd(q, k, v, causal=True, scale=0.2)
    for h in range(Hq):
        np.testing.assert_array_equal(o[0, h, 0], v[0, h, 0])
        np.testing.assert_allclose(lse[0, h, 0], 0.2 * math.fsum(q[0, h, 0] * k[0, h, 0]),
                                   rtol=0, atol=1e-13)


def pin_matches_torch_sdpa(fwd):
    """Against PyTorch's scaled_dot_product_attention in fp64 on the CPU (the
    library routine the wiki note names) with an explicit boolean mask and
    enable_gqa; LSE against torch.logsumexp of the masked scaled scores."""
    import torch
    import torch.nn.functional as F

    for (B, Hq, Hkv, N, d, causal, sl, seed) in [
        (2, 4, 2, 33, 16, False, [33, 7], 21),
        (2, 6, 3, 40, 8, True, None, 22),
        (3, 2, 1, 25, 12, True, [25, 1, 13], 23),
        (1, 8, 8, 64, 32, False, None, 24),
    ]:
        q, k, v = _rng_inputs(seed, B, Hq, Hkv, N, d, 1.5)
        scale = 1.0 / math.sqrt(d)
        sln = None if sl is None else np.array(sl, np.int32)
        o, lse = fwd(q, k, v, causal=causal, scale=scale, seqlens=sln)
        i = torch.arange(N)[:, None]
        j = torch.arange(N)[None, :]
        lens = torch.tensor(sl if sl is not None else [N] * B)
        allowed = (j[None] < lens[:, None, None])  # [B, N, N]
        if causal:
            allowed = allowed & (j <= i)[None]
        allowed = allowed[:, None]  # broadcast over heads
        tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
        ref = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=allowed, scale=scale,
                                             enable_gqa=True)
        np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
        kk = tk.repeat_interleave(Hq // Hkv, dim=1)
        s = torch.matmul(tq, kk.transpose(-1, -2)) * scale
        s = s.masked_fill(~allowed, float("-inf"))
        np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)


def _brute(q, k, v, causal, scale, seqlens, bottom_right=False):
    """Two passes per row in plain Python with math.exp: max, then sums."""
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, Nq))
    for b in range(B):
        L = Nk if seqlens is None else int(seqlens[b])
        off = L - Nq if bottom_right else 0
        for h in range(Hq):
            g = h // (Hq // Hkv)
            for i in range(Nq):
                vis = [j for j in range(Nk) if j < L and (not causal or j <= i + off)]
                s = {j: scale * math.fsum(float(q[b, h, i, c]) * float(k[b, g, j, c])
                                          for c in range(d)) for j in vis}
                mx = max(s.values())
                w = {j: math.exp(s[j] - mx) for j in vis}
                z = math.fsum(w.values())
                for c in range(d):
                    o[b, h, i, c] = math.fsum(w[j] * float(v[b, g, j, c]) for j in vis) / z
                lse[b, h, i] = mx + math.log(z)
    return o, lse


def pin_brute_force(fwd):
    """Tiny cases against a pure-Python two-pass softmax (max pass, then
    exp/sum pass) with masks and GQA."""
    for (B, Hq, Hkv, N, d, causal, sl, seed) in [
        (1, 2, 1, 7, 3, False, None, 31),
        (2, 4, 2, 9, 2, True, [9, 4], 32),
        (2, 3, 3, 6, 4, False, [2, 6], 33),
    ]:
        q, k, v = _rng_inputs(seed, B, Hq, Hkv, N, d, 2.5)
        sln = None if sl is None else np.array(sl, np.int32)
        o, lse = fwd(q, k, v, causal=causal, scale=0.61, seqlens=sln)
        ob, lb = _brute(q, k, v, causal, 0.61, sln)
        np.testing.assert_allclose(o, ob, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-13)


def pin_key_permutation_invariance(fwd):
    """Non-causal attention is a sum over keys: permuting K and V rows
    jointly (with no padding) leaves O and LSE unchanged."""
    B, Hq, Hkv, N, d = 1, 4, 2, 31, 7
    q, k, v = _rng_inputs(41, B, Hq, Hkv, N, d)
    perm = np.random.default_rng(42).permutation(N)
    o1, l1 = fwd(q, k, v, causal=False, scale=0.33)
    o2, l2 = fwd(q, k[:, :, perm], v[:, :, perm], causal=False, scale=0.33)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def pin_linear_in_v(fwd):
    """O is linear in V for fixed Q, K: O(aV1 + V2) = a O(V1) + O(V2)."""
    B, Hq, Hkv, N, d = 2, 2, 2, 19, 5
    q, k, v1 = _rng_inputs(43, B, Hq, Hkv, N, d)
    v2 = np.random.default_rng(44).standard_normal(v1.shape)
    sl = np.array([19, 11], np.int32)
    for causal in (False, True):
        a, _ = fwd(q, k, v1, causal=causal, scale=0.5, seqlens=sl)
        b, _ = fwd(q, k, v2, causal=causal, scale=0.5, seqlens=sl)
        c, _ = fwd(q, k, 3.0 * v1 + v2, causal=causal, scale=0.5, seqlens=sl)
        np.testing.assert_allclose(c, 3.0 * a + b, rtol=0, atol=1e-12)


def pin_shift_invariance(fwd):
    """Adding the same constant to every score of a row leaves P (so O)
    unchanged and moves LSE by that constant.  The shift is made through an
    extra feature (q gets c, k gets 1) and is large enough (800) that exp of
    an unshifted score overflows fp64: the row max must be subtracted."""
    B, Hq, Hkv, N, d = 1, 2, 2, 23, 4
    q, k, v = _rng_inputs(45, B, Hq, Hkv, N, d)
    scale = 0.5
    shift = 800.0
    q2 = np.concatenate([q, np.full((B, Hq, N, 1), shift / scale)], axis=-1)
    k2 = np.concatenate([k, np.ones((B, Hkv, N, 1))], axis=-1)
    v2 = np.concatenate([v, np.zeros((B, Hkv, N, 1))], axis=-1)
    for causal in (False, True):
        o1, l1 = fwd(q, k, v, causal=causal, scale=scale)
        o2, l2 = fwd(q2, k2, v2, causal=causal, scale=scale)
        assert np.all(np.isfinite(o2)) and np.all(np.isfinite(l2))
        np.testing.assert_allclose(o2[..., :d], o1, rtol=0, atol=1e-11)
        np.testing.assert_allclose(l2 - shift, l1, rtol=0, atol=1e-10)


def pin_fully_masked_row(fwd):
    """A row with no visible key (len_b = 0) gives O = 0 and LSE = -inf."""
    q, k, v = _rng_inputs(46, 2, 1, 1, 5, 3)
    o, lse = fwd(q, k, v, causal=False, scale=1.0, seqlens=np.array([0, 5], np.int32))
    assert np.all(o[0] == 0.0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(lse[1]))


def pin_row_subset(fwd):
    """Computing a subset of query rows gives exactly those rows of the full
    result (rows are independent)."""
    B, Hq, Hkv, N, d = 2, 4, 1, 45, 6
    q, k, v = _rng_inputs(47, B, Hq, Hkv, N, d)
    rows = np.stack([np.sort(np.random.default_rng(48 + i).choice(N, 10, replace=False))
                     for i in range(B * Hq)])
    for causal in (False, True):
        of, lf = fwd(q, k, v, causal=causal, scale=0.4)
        os_, ls = fwd(q, k, v, causal=causal, scale=0.4, rows=rows)
        for bh in range(B * Hq):
            b, h = divmod(bh, Hq)
            np.testing.assert_array_equal(os_[b, h], of[b, h, rows[bh]])
            np.testing.assert_array_equal(ls[b, h], lf[b, h, rows[bh]])


def pin_input_encodings_agree(fwd):
    """bf16 bit patterns, their fp32 values and their fp64 values are the
    same numbers, so all three input encodings give identical results."""
    rng = np.random.default_rng(49)
    x = rng.standard_normal((3, 1, 2, 24, 8)).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)  # truncation: any bf16 values will do
    f32 = (bits.astype(np.uint32) << 16).view(np.float32)
    res = [fwd(a[0], a[1], a[2], causal=True, scale=0.35)
           for a in (bits, f32, f32.astype(np.float64))]
    for o, l in res[1:]:
        np.testing.assert_array_equal(o, res[0][0])
        np.testing.assert_array_equal(l, res[0][1])


def pin_e4m3_codes(fwd):
    """FP8 E4M3 inputs (uint8 codes).  Through V: one visible key makes
    O = V_0, so O shows the decoded value of every non-NaN code, which must
    equal torch's float8_e4m3fn widening and, for a few codes, the values
    worked out by hand from the format (bias 7, 3 mantissa bits, subnormals
    m * 2^-9).  Through Q: one key of value 1 makes LSE = scale * q."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    codes = codes[(codes & 0x7F) != 0x7F]  # S.1111.111 is NaN
    n = codes.size
    zeros = np.zeros((1, 1, 1, n), np.uint8)
    o, _ = fwd(zeros, zeros, codes.reshape(1, 1, 1, n), causal=False, scale=1.0)
    lib = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(o.ravel(), lib)
    by_hand = {0x00: 0.0, 0x38: 1.0, 0xB8: -1.0, 0x7E: 448.0, 0x01: 2.0 ** -9,
               0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x3C: 1.5, 0x40: 2.0, 0x46: 3.5, 0x4B: 5.5}
    for c, val in by_hand.items():
        assert o.ravel()[list(codes).index(c)] == val, hex(c)
    one = np.full((1, 1, 1, 1), 0x38, np.uint8)
    q = codes.reshape(1, 1, n, 1)
    _, lse = fwd(q, one, one, causal=False, scale=0.5)
    np.testing.assert_array_equal(lse.ravel(), 0.5 * lib)


def pin_e4m3_matches_decoded_fp64(fwd):
    """Attention on E4M3 codes equals attention on their values in fp64."""
    import torch
    rng = np.random.default_rng(57)
    codes = rng.integers(0, 256, size=(3, 2, 1, 20, 16), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x30  # no NaN codes
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    a = fwd(codes[0], codes[1][:, :1], codes[2][:, :1], causal=True, scale=0.01)
    b = fwd(vals[0], vals[1][:, :1], vals[2][:, :1], causal=True, scale=0.01)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def pin_cross_length_matches_torch_sdpa(fwd):
    """Nq query rows against Nk keys (the decode shape), causal aligned to the
    end of each sequence's keys, against torch SDPA in fp64 with the same
    explicit mask, and against the pure-Python two-pass softmax."""
    import torch
    import torch.nn.functional as F

    for (B, Hq, Hkv, Nq, Nk, d, causal, sl, seed) in [
        (2, 4, 2, 1, 37, 8, True, [37, 9], 51),
        (2, 4, 1, 3, 50, 16, True, [50, 4], 52),
        (1, 2, 2, 5, 23, 4, False, None, 53),
        (3, 6, 3, 2, 40, 12, True, None, 54),
    ]:
        rng = np.random.default_rng(seed)
        q = rng.standard_normal((B, Hq, Nq, d))
        k = rng.standard_normal((B, Hkv, Nk, d)) * 1.7
        v = rng.standard_normal((B, Hkv, Nk, d))
        sln = None if sl is None else np.array(sl, np.int32)
        o, lse = fwd(q, k, v, causal=causal, scale=0.4, seqlens=sln, causal_bottom_right=True)
        lens = torch.tensor(sl if sl is not None else [Nk] * B)
        i = torch.arange(Nq)[None, :, None]
        j = torch.arange(Nk)[None, None, :]
        allowed = j < lens[:, None, None]
        if causal:
            allowed = allowed & (j <= i + (lens - Nq)[:, None, None])
        allowed = allowed[:, None]
        tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
        dead = ~allowed.any(-1)  # rows with no visible key
        ref = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=allowed, scale=0.4,
                                             enable_gqa=True)
        ref = torch.where(dead[..., None], torch.zeros_like(ref), ref)
        np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
        ob, lb = _brute(q, k, v, causal, 0.4, sln, bottom_right=True)
        np.testing.assert_allclose(o, ob, rtol=0, atol=1e-13)
        live = np.isfinite(lb)
        np.testing.assert_allclose(lse[live], lb[live], rtol=0, atol=1e-13)
        assert np.all(np.isneginf(lse[~live]))


def pin_single_query_is_last_causal_row(fwd):
    """A single query at the end of a sequence (causal, bottom-right) sees
    every key, so it equals the last row of the square causal forward, and
    its LSE is the log-sum-exp of that whole row."""
    B, Hq, Hkv, N, d = 2, 4, 2, 33, 8
    q, k, v = _rng_inputs(55, B, Hq, Hkv, N, d, 1.3)
    o_full, l_full = fwd(q, k, v, causal=True, scale=0.3)
    o1, l1 = fwd(np.ascontiguousarray(q[:, :, -1:]), k, v, causal=True, scale=0.3,
                 causal_bottom_right=True)
    np.testing.assert_allclose(o1[:, :, 0], o_full[:, :, -1], rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1[:, :, 0], l_full[:, :, -1], rtol=0, atol=1e-13)
    # with key lengths, the query sits at position len_b - 1
    sl = np.array([33, 12], np.int32)
    o1, l1 = fwd(np.ascontiguousarray(q[:, :, 11:12]), k, v, causal=True, scale=0.3,
                 seqlens=np.array([12, 12], np.int32), causal_bottom_right=True)
    o_s, l_s = fwd(q, k, v, causal=True, scale=0.3, seqlens=sl)
    np.testing.assert_allclose(o1[1, :, 0], o_s[1, :, 11], rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1[1, :, 0], l_s[1, :, 11], rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------
# Backward pins: fn is a pair (fwd, bwd) for these.
# ---------------------------------------------------------------------------
def _bwd_inputs(seed, B, Hq, Hkv, N, d):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, Hq, N, d)), rng.standard_normal((B, Hkv, N, d)) * 1.4,
            rng.standard_normal((B, Hkv, N, d)), rng.standard_normal((B, Hq, N, d)))


def pin_bwd_matches_torch_autograd(fwd, bwd):
    """Gradients against torch autograd through scaled_dot_product_attention
    in fp64 with the same explicit mask and enable_gqa."""
    import torch
    import torch.nn.functional as F
    for (B, Hq, Hkv, N, d, causal, sl, seed) in [
        (2, 4, 2, 21, 8, True, [21, 6], 61),
        (1, 6, 3, 30, 16, False, [11], 62),
        (2, 2, 2, 17, 4, True, None, 63),
    ]:
        q, k, v, do = _bwd_inputs(seed, B, Hq, Hkv, N, d)
        sln = None if sl is None else np.array(sl, np.int32)
        dq, dk, dv = bwd(q, k, v, do, causal=causal, scale=0.35, seqlens=sln)
        i = torch.arange(N)[:, None]
        j = torch.arange(N)[None, :]
        lens = torch.tensor(sl if sl is not None else [N] * B)
        allowed = j[None] < lens[:, None, None]
        if causal:
            allowed = allowed & (j <= i)[None]
        tq, tk, tv = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
        o = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=allowed[:, None], scale=0.35,
                                           enable_gqa=True)
        o.backward(torch.from_numpy(do))
        np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=0, atol=1e-11)


def pin_bwd_finite_differences(fwd, bwd):
    """Central differences of L = sum(dO * O) computed with the forward
    oracle, along random directions in Q, K and V."""
    B, Hq, Hkv, N, d = 1, 4, 2, 13, 6
    q, k, v, do = _bwd_inputs(64, B, Hq, Hkv, N, d)
    sl = np.array([10], np.int32)
    dq, dk, dv = bwd(q, k, v, do, causal=True, scale=0.5, seqlens=sl)

    def loss(qq, kk, vv):
        o, _ = fwd(qq, kk, vv, causal=True, scale=0.5, seqlens=sl)
        return float(np.sum(do * o))

    rng = np.random.default_rng(65)
    h = 1e-5
    for which, grad in (("q", dq), ("k", dk), ("v", dv)):
        for _ in range(3):
            u = rng.standard_normal(grad.shape)
            args = {"q": q, "k": k, "v": v}
            plus = dict(args)
            minus = dict(args)
            plus[which] = args[which] + h * u
            minus[which] = args[which] - h * u
            fd = (loss(plus["q"], plus["k"], plus["v"]) - loss(minus["q"], minus["k"], minus["v"])) / (2 * h)
            assert abs(fd - float(np.sum(grad * u))) <= 1e-6 * max(1.0, abs(fd)), which


def pin_bwd_key_gradients_sum_to_zero(fwd, bwd):
    """Adding one vector to every key shifts each row's scores by a constant,
    which the softmax ignores, so the key gradients of each (batch, kv head)
    sum to zero; keys that no query sees get zero gradients, and so do query
    rows that see no key."""
    B, Hq, Hkv, N, d = 2, 4, 2, 25, 8
    q, k, v, do = _bwd_inputs(66, B, Hq, Hkv, N, d)
    sl = np.array([25, 9], np.int32)
    for causal in (False, True):
        dq, dk, dv = bwd(q, k, v, do, causal=causal, scale=0.4, seqlens=sl)
        np.testing.assert_allclose(dk.sum(axis=2), 0.0, rtol=0, atol=1e-12)
        assert np.all(dk[1, :, 9:] == 0.0) and np.all(dv[1, :, 9:] == 0.0)
    dq, dk, dv = bwd(q, k, v, do, causal=False, scale=0.4, seqlens=np.array([25, 0], np.int32))
    assert np.all(dq[1] == 0.0) and np.all(dk[1] == 0.0) and np.all(dv[1] == 0.0)


BWD_PINS = [pin_bwd_matches_torch_autograd, pin_bwd_finite_differences,
            pin_bwd_key_gradients_sum_to_zero]


ALL_PINS = [
    pin_golden, pin_probs_are_a_row_softmax, pin_constant_v, pin_single_visible_key,
    pin_causal_first_row, pin_matches_torch_sdpa, pin_brute_force,
    pin_key_permutation_invariance, pin_linear_in_v, pin_shift_invariance,
    pin_fully_masked_row, pin_row_subset, pin_input_encodings_agree,
    pin_cross_length_matches_torch_sdpa, pin_single_query_is_last_causal_row,
    pin_e4m3_codes, pin_e4m3_matches_decoded_fp64,
]
