"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Small shapes span several tiles and ragged tails (every row checked); the five
workloads run at their full sizes in the launch configuration the benchmark
uses, checked on every row where the oracle is quick and on seeded samples of
rows where it is not.
"""
import numpy as np
import pytest

from exact_io_aware_92_b200 import workloads as wl
from parity_helpers import (LSE_TOL_BF16, O_TOL_BF16, TOL_F32, compare, derived_o_bound,
                            gather_rows, reference, run_bf16, run_f32)

pytestmark = pytest.mark.gpu


def _case(B, Hq, Hkv, N, d, causal, seed, seqlens=None, k_scale=1.0, derived_bound=False):
    inp = wl.draw(B, Hq, Hkv, N, d, seed, k_scale=k_scale)
    if seqlens is not None:
        inp.seqlens = np.asarray(seqlens, dtype=np.int32)
    scale = 1.0 / np.sqrt(d)
    o, lse = run_bf16(inp, causal=causal, scale=scale)
    o_bound = None
    if derived_bound:
        o_ref, lse_ref, p = reference(inp, causal=causal, scale=scale, return_probs=True)
        o_bound = derived_o_bound(inp, p, o_ref, float(np.float32(scale)))
    else:
        o_ref, lse_ref = reference(inp, causal=causal, scale=scale)
    return compare(o, lse, o_ref, lse_ref, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16,
                   what=f"B{B} Hq{Hq} Hkv{Hkv} N{N} d{d} causal{causal} sl{seqlens}",
                   o_bound=o_bound)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 127, 128, 129, 255, 256, 257, 383, 640])
def test_ragged_lengths(N, d, causal):
    _case(1, 2, 1, N, d, causal, seed=1000 + N)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_key_padding_edges(d, causal):
    # lengths at 0 (no visible key), 1, around one tile, and the full N
    _case(7, 2, 2, 512, d, causal, seed=77, seqlens=[0, 1, 63, 127, 128, 129, 512])


@pytest.mark.parametrize("group", [1, 4, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_groups(group, causal):
    _case(2, 8, 8 // group, 300, 128, causal, seed=90 + group)


def test_sharpened_scores():
    # K scaled by 8 (a stress input, not one of the workloads): near one-hot
    # rows make O a single V row, often with |O| >= 4 where bf16 itself is
    # coarser than 1.5e-2.  1.5e-2 stays the floor; an element beyond it
    # must lie within the bound derived from the kernel's roundings and the
    # oracle's weights, and at most 1e-4 of the elements may need that.
    _, _, n1 = _case(1, 4, 2, 700, 128, True, seed=5, k_scale=8.0, derived_bound=True)
    _, _, n2 = _case(1, 4, 2, 700, 64, False, seed=6, k_scale=8.0, derived_bound=True)
    print(f"elements beyond 1.5e-2, each within its derived bound: {n1 + n2}")


def test_tiny_bf16():
    w = wl.TINY
    inp = wl.draw_workload(w)
    o, lse = run_bf16(inp, causal=w.causal, scale=w.scale)
    o_ref, lse_ref = reference(inp, causal=w.causal, scale=w.scale)
    compare(o, lse, o_ref, lse_ref, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16, what=w.name)


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_fp32_check_mode(causal):
    w = wl.TINY
    inp = wl.draw_workload(w)
    o, lse = run_f32(inp, causal=causal, scale=w.scale)
    o_ref, lse_ref = reference(inp, causal=causal, scale=w.scale)
    compare(o, lse, o_ref, lse_ref, o_tol=TOL_F32, lse_tol=TOL_F32, what="tiny fp32")


@pytest.mark.parametrize("d", [64, 128])
def test_fp32_check_mode_masks(d):
    inp = wl.draw(2, 4, 2, 300, d, seed=321)
    inp.seqlens = np.array([300, 77], dtype=np.int32)
    for causal in (False, True):
        o, lse = run_f32(inp, causal=causal, scale=1.0 / np.sqrt(d))
        o_ref, lse_ref = reference(inp, causal=causal, scale=1.0 / np.sqrt(d))
        compare(o, lse, o_ref, lse_ref, o_tol=TOL_F32, lse_tol=TOL_F32, what=f"fp32 d{d}")


@pytest.mark.parametrize("w", [wl.GPT2, wl.BERT], ids=lambda w: w.name)
def test_full_workload_every_row(w):
    inp = wl.draw_workload(w)
    o, lse = run_bf16(inp, causal=w.causal, scale=w.scale)
    o_ref, lse_ref = reference(inp, causal=w.causal, scale=w.scale)
    compare(o, lse, o_ref, lse_ref, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16, what=w.name)


@pytest.mark.parametrize("w", [wl.LLAMA_GQA, wl.LONG], ids=lambda w: w.name)
def test_full_workload_sampled_rows(w):
    inp = wl.draw_workload(w)
    o, lse = run_bf16(inp, causal=w.causal, scale=w.scale)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    rows = wl.sample_rows(w)
    # always include the first and last rows of every head
    rows[:, 0] = 0
    rows[:, -1] = w.N - 1
    rows.sort(axis=1)
    o_ref, lse_ref = reference(inp, causal=w.causal, scale=w.scale, rows=rows)
    og, lg = gather_rows(o, lse, rows)
    compare(og, lg, o_ref, lse_ref, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16, what=w.name)


def test_llama_gqa_every_row_of_one_group():
    # The contract launch (B2 Hq32 Hkv8 N8192 d128, K x 2) with every output
    # row of one (batch, kv head) group checked: its four query heads' O and
    # LSE depend only on that group's Q, K and V.
    w = wl.LLAMA_GQA
    inp = wl.draw_workload(w)
    o, lse = run_bf16(inp, causal=w.causal, scale=w.scale)
    b, g = 0, 3
    G = w.Hq // w.Hkv
    hs = slice(g * G, (g + 1) * G)
    part = wl.Inputs(q_bits=inp.q_bits[b:b + 1, hs], k_bits=inp.k_bits[b:b + 1, g:g + 1],
                     v_bits=inp.v_bits[b:b + 1, g:g + 1], seqlens=None)
    o_ref, lse_ref = reference(part, causal=w.causal, scale=w.scale)
    compare(o[b:b + 1, hs], lse[b:b + 1, hs], o_ref, lse_ref, o_tol=O_TOL_BF16,
            lse_tol=LSE_TOL_BF16, what=f"{w.name} group (b={b}, kv head {g})")


@pytest.mark.parametrize("causal,lens", [(True, None), (False, [4096, 2500, 1, 3333])])
def test_long_d64_sampled_rows(causal, lens):
    # d = 64 rotates three S buffers over both Q tiles' products: units of up
    # to 32 key tiles, many units per CTA, K x 2 for more rescales.
    B = 4
    inp = wl.draw(B, 8, 2, 4096, 64, seed=1900 + int(causal), k_scale=2.0)
    if lens is not None:
        inp.seqlens = np.asarray(lens, dtype=np.int32)
    o, lse = run_bf16(inp, causal=causal, scale=0.125)
    assert np.all(np.isfinite(o))
    w = wl.Workload("long_d64", B, 8, 2, 4096, 64, causal, seed=1900)
    rows = wl.sample_rows(w, 64)
    rows[:, 0] = 0
    rows[:, -1] = 4095
    rows.sort(axis=1)
    o_ref, lse_ref = reference(inp, causal=causal, scale=0.125, rows=rows)
    og, lg = gather_rows(o, lse, rows)
    compare(og, lg, o_ref, lse_ref, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16,
            what=f"long d64 causal={causal}")


@pytest.mark.parametrize("B,H,N,d,causal", [(1, 16, 16384, 128, False), (4, 16, 16384, 64, True)])
def test_kv_beyond_l2_sampled_rows(B, H, N, d, causal):
    # 134 and 268 MB of K/V, more than the 126 MB L2: query tiles of a head
    # read its K/V tiles again from DRAM; many units per CTA at d = 64.
    inp = wl.draw(B, H, H, N, d, seed=2100 + d, k_scale=2.0)
    scale = 1.0 / np.sqrt(d)
    o, lse = run_bf16(inp, causal=causal, scale=scale)
    assert np.all(np.isfinite(o))
    w = wl.Workload("kv_beyond_l2", B, H, H, N, d, causal, seed=2100 + d)
    rows = wl.sample_rows(w, 24)
    rows[:, 0] = 0
    rows[:, -1] = N - 1
    rows.sort(axis=1)
    o_ref, lse_ref = reference(inp, causal=causal, scale=scale, rows=rows)
    og, lg = gather_rows(o, lse, rows)
    compare(og, lg, o_ref, lse_ref, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16,
            what=f"K/V beyond L2 d{d} causal={causal}")


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", [
    (2, 32, 8, 8000, 128, True),     # 8000 = 31 * 256 + 64: 64 rows in Q tile 0, none in Q tile 1
    (2, 16, 4, 6001, 128, False),    # 6001 = 23 * 256 + 113: Q tile 1 of the last unit is empty
    (1, 8, 2, 12345, 64, True),      # d = 64 three-buffer sequence with a ragged tail
    (3, 8, 8, 10184, 64, False),     # 10184 = 39 * 256 + 200: Q tile 1 holds 72 rows
])
def test_ragged_length_at_scale_sampled_rows(B, Hq, Hkv, N, d, causal):
    # Many units per CTA, a partial last round of the unit order, and a last
    # unit whose Q and key tiles are cut short: rows around every tail
    # boundary are always checked, the rest sampled.
    inp = wl.draw(B, Hq, Hkv, N, d, seed=2300 + N % 97, k_scale=2.0)
    scale = 1.0 / np.sqrt(d)
    o, lse = run_bf16(inp, causal=causal, scale=scale)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    rng = np.random.default_rng(2300 + N)
    tail = [N - 257, N - 256, N - 255, N - 129, N - 128, N - 127, N - 2, N - 1]
    rows = np.empty((B * Hq, 1 + 16 + len(tail)), dtype=np.int64)
    for bh in range(B * Hq):
        rows[bh] = np.sort(np.concatenate(
            [[0], rng.choice(np.arange(1, N - 300), size=16, replace=False), tail]))
    o_ref, lse_ref = reference(inp, causal=causal, scale=scale, rows=rows)
    og, lg = gather_rows(o, lse, rows)
    compare(og, lg, o_ref, lse_ref, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16,
            what=f"ragged N={N} d{d} causal={causal}")


def test_deterministic():
    inp = wl.draw(2, 8, 2, 1000, 128, seed=55)
    a = run_bf16(inp, causal=True, scale=0.088)
    b = run_bf16(inp, causal=True, scale=0.088)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
