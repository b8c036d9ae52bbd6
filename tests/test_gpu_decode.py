"""Split-KV decode forward (fa_fwd_decode) vs the fp64 oracle with queries at
the end of their sequences, element by element."""
import numpy as np
import pytest

from exact_io_aware_92_b200 import workloads as wl
from parity_helpers import LSE_TOL_BF16, O_TOL_BF16, compare, to_device_bf16

pytestmark = pytest.mark.gpu

import oracle  # noqa: E402


def run_decode(inp, *, causal, scale, num_splits=0):
    import torch
    from exact_io_aware_92_b200 import attention
    q, k, v = (to_device_bf16(x) for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    sl = None if inp.seqlens is None else torch.from_numpy(inp.seqlens).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = attention.fwd_decode(q, k, v, causal=causal, scale=scale, seqlens=sl,
                                  num_splits=num_splits, status=status)
    assert attention.check_status(status) == 0
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def ref_decode(inp, *, causal, scale):
    return oracle.attention_forward(inp.q_bits, inp.k_bits, inp.v_bits, causal=causal,
                                    scale=float(np.float32(scale)), seqlens=inp.seqlens,
                                    causal_bottom_right=True)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Nk", [1, 17, 64, 65, 129, 1000, 4097])
def test_single_query_lengths(Nk, d):
    inp = wl.draw(2, 8, 2, Nk, d, seed=600 + Nk, nq=1)
    o, lse = run_decode(inp, causal=True, scale=1 / np.sqrt(d))
    o_r, l_r = ref_decode(inp, causal=True, scale=1 / np.sqrt(d))
    compare(o, lse, o_r, l_r, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16, what=f"Nk{Nk} d{d}")


# Up to 16 query rows per kv head take the tensor-core kernel with keys on the
# tensor-memory lanes (4, 8 or 16 row slots); 17 to 128 the one with rows on
# the lanes: (4, 5) and (8, 3) give 20 and 24.
@pytest.mark.parametrize("splits", [1, 3, 7, 0])
@pytest.mark.parametrize("group,nq", [(1, 1), (4, 1), (8, 1), (4, 3), (1, 5), (4, 4), (4, 5),
                                      (8, 3)])
def test_groups_rows_and_splits(group, nq, splits):
    inp = wl.draw(3, 8, 8 // group, 2000, 128, seed=700 + group * 10 + nq, nq=nq)
    inp.seqlens = np.array([2000, 1, 777], dtype=np.int32)
    for causal in (False, True):
        o, lse = run_decode(inp, causal=causal, scale=0.09, num_splits=splits)
        o_r, l_r = ref_decode(inp, causal=causal, scale=0.09)
        compare(o, lse, o_r, l_r, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16,
                what=f"G{group} nq{nq} splits{splits} causal{causal}")


def test_empty_and_short_caches():
    inp = wl.draw(4, 4, 2, 300, 64, seed=801, nq=2)
    inp.seqlens = np.array([0, 1, 2, 300], dtype=np.int32)
    o, lse = run_decode(inp, causal=True, scale=0.125, num_splits=4)
    o_r, l_r = ref_decode(inp, causal=True, scale=0.125)
    compare(o, lse, o_r, l_r, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16, what="short caches")


def test_decode_workload_every_row():
    w = wl.DECODE
    inp = wl.draw_workload(w)
    o, lse = run_decode(inp, causal=w.causal, scale=w.scale)
    o_r, l_r = ref_decode(inp, causal=w.causal, scale=w.scale)
    compare(o, lse, o_r, l_r, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16, what=w.name)


def test_decode_matches_last_row_of_full_forward():
    """A single query at the end of a sequence equals the last causal row of
    the tensor-core forward over the same keys (two kernels, same answer
    within rounding)."""
    import torch
    from exact_io_aware_92_b200 import attention
    full = wl.draw(2, 8, 2, 1000, 128, seed=802)
    q, k, v = (to_device_bf16(x) for x in (full.q_bits, full.k_bits, full.v_bits))
    o_full, l_full = attention.fwd(q, k, v, causal=True, scale=0.088)
    o_dec, l_dec = attention.fwd_decode(q[:, :, -1:].contiguous(), k, v, causal=True, scale=0.088)
    torch.cuda.synchronize()
    assert torch.allclose(o_dec[:, :, 0].float(), o_full[:, :, -1].float(), atol=2e-2)
    assert torch.allclose(l_dec[:, :, 0], l_full[:, :, -1], atol=1e-3)


@pytest.mark.parametrize("splits", [0, 5, 1])
@pytest.mark.parametrize("group,nq", [(4, 3), (8, 2)])
def test_d64_twelve_and_sixteen_rows(group, nq, splits):
    # d = 64 with 12 and 16 query rows per kv head: the tensor-core kernel's
    # 16-slot instance, whose PV product stacks the two key halves (N = 32).
    inp = wl.draw(2, 8, 8 // group, 1500, 64, seed=900 + group * 10 + nq, nq=nq)
    inp.seqlens = np.array([1500, 613], dtype=np.int32)
    for causal in (False, True):
        o, lse = run_decode(inp, causal=causal, scale=0.125, num_splits=splits)
        o_r, l_r = ref_decode(inp, causal=causal, scale=0.125)
        compare(o, lse, o_r, l_r, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16,
                what=f"d64 G{group} nq{nq} splits{splits} causal{causal}")


@pytest.mark.parametrize("splits", [1, 2, 0])
def test_many_short_caches_per_cta(splits):
    # 40 sequences x 2 kv heads with short, ragged caches (some empty): a
    # CTA's share of the tiles spans many (batch, kv head) pieces.
    B = 40
    inp = wl.draw(B, 8, 2, 300, 128, seed=950 + splits, nq=1)
    rng = np.random.default_rng(951)
    lens = rng.integers(0, 301, size=B).astype(np.int32)
    lens[[3, 17, 29]] = 0
    inp.seqlens = lens
    o, lse = run_decode(inp, causal=True, scale=0.088, num_splits=splits)
    o_r, l_r = ref_decode(inp, causal=True, scale=0.088)
    compare(o, lse, o_r, l_r, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16,
            what=f"B{B} short caches splits{splits}")


# Rows on the tensor-memory lanes (17 to 128 query rows per kv head): 24, 32,
# 64 and 128 rows, with ragged and empty caches, both head dims, forced
# splits (several pieces per CTA, several CTAs per piece) and the automatic
# split; beyond 128 rows (8 x 17 = 136) the CUDA-core kernel.
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("group,nq", [(8, 3), (8, 4), (4, 16), (16, 8), (8, 17)])
@pytest.mark.parametrize("splits", [0, 3])
def test_rows_on_lanes(group, nq, splits, d):
    Hkv = 2
    inp = wl.draw(3, group * Hkv, Hkv, 1500, d, seed=1000 + group * 10 + nq + d, nq=nq)
    inp.seqlens = np.array([1500, 0, 333], dtype=np.int32)
    for causal in (False, True):
        o, lse = run_decode(inp, causal=causal, scale=1 / np.sqrt(d), num_splits=splits)
        o_r, l_r = ref_decode(inp, causal=causal, scale=1 / np.sqrt(d))
        compare(o, lse, o_r, l_r, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16,
                what=f"d{d} G{group} nq{nq} splits{splits} causal{causal}")


def test_rows_on_lanes_gqa8_decode_workload():
    # group size 8 with 4 query rows per sequence (speculative or chunked
    # decode): 8 query heads per kv head x 4 = 32 rows per kv head; every row
    w = wl.DECODE_NQ4
    inp = wl.draw_workload(w)
    o, lse = run_decode(inp, causal=w.causal, scale=w.scale)
    o_r, l_r = ref_decode(inp, causal=w.causal, scale=w.scale)
    compare(o, lse, o_r, l_r, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16, what=w.name)


@pytest.mark.parametrize("lens", [[0, 0, 0], [1, 1, 1], [0, 1, 129]])
def test_rows_kernel_empty_and_one_key_caches(lens):
    # 32 query rows per kv head (rows on the lanes) with caches that are
    # empty or hold one key: most CTAs get no tile, some rows see no key.
    inp = wl.draw(3, 16, 2, 200, 128, seed=1200 + sum(lens), nq=4)
    inp.seqlens = np.array(lens, dtype=np.int32)
    o, lse = run_decode(inp, causal=True, scale=0.088)
    o_r, l_r = ref_decode(inp, causal=True, scale=0.088)
    compare(o, lse, o_r, l_r, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16, what=f"lens {lens}")


def test_decode_repeats_bitwise_and_on_other_streams():
    # Each CTA's share covers fixed keys and the merge visits the partials in
    # a fixed order: repeated calls, on one stream or on another, give
    # identical bits.
    import torch
    from exact_io_aware_92_b200 import attention
    inp = wl.draw(8, 32, 4, 6000, 128, seed=1190, nq=4)
    inp.seqlens = np.random.default_rng(1191).integers(3000, 6001, size=8).astype(np.int32)
    q, k, v = (to_device_bf16(x) for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    sl = torch.from_numpy(inp.seqlens).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    for _ in range(3):
        outs.append(attention.fwd_decode(q, k, v, causal=True, scale=0.088, seqlens=sl,
                                         status=status))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(2):
            outs.append(attention.fwd_decode(q, k, v, causal=True, scale=0.088, seqlens=sl,
                                             status=status))
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert attention.check_status(status) == 0
    for o, lse in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(lse, outs[0][1])
    o_r, l_r = ref_decode(inp, causal=True, scale=0.088)
    compare(outs[0][0].float().cpu().numpy().astype(np.float64),
            outs[0][1].cpu().numpy().astype(np.float64), o_r, l_r, o_tol=O_TOL_BF16,
            lse_tol=LSE_TOL_BF16, what="repeated calls")
