"""Packed variable-length forward (fa_fwd_varlen) vs the fp64 oracle run per
sequence on the same values."""
import numpy as np
import pytest

from exact_io_aware_92_b200 import workloads as wl
from parity_helpers import LSE_TOL_BF16, O_TOL_BF16, compare

pytestmark = pytest.mark.gpu

import oracle  # noqa: E402


def run_varlen(q_bits, k_bits, v_bits, lengths, *, causal, scale):
    import torch
    from exact_io_aware_92_b200 import attention
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).cuda()  # noqa
    cu = torch.from_numpy(wl.cu_seqlens(lengths)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = attention.fwd_varlen(to(q_bits), to(k_bits), to(v_bits), cu, int(max(lengths)),
                                  causal=causal, scale=scale, status=status)
    assert attention.check_status(status) == 0
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def check_against_padded(inp, lengths, *, causal, scale, what):
    """inp holds padded [B, H, N, d] draws; sequence b uses its first L_b rows."""
    qp, kp, vp = (wl.pack(x, lengths) for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    o, lse = run_varlen(qp, kp, vp, lengths, causal=causal, scale=scale)
    cu = wl.cu_seqlens(lengths)
    for b, L in enumerate(lengths):
        if L == 0:
            continue
        sl = lambda x: np.ascontiguousarray(x[b:b + 1, :, :L, :])  # noqa: E731
        o_r, l_r = oracle.attention_forward(sl(inp.q_bits), sl(inp.k_bits), sl(inp.v_bits),
                                            causal=causal, scale=float(np.float32(scale)))
        og = np.transpose(o[cu[b]:cu[b + 1]], (1, 0, 2))[None]
        lg = lse[:, cu[b]:cu[b + 1]][None]
        compare(og, lg, o_r, l_r, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16, what=f"{what} seq {b}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_packed_sequences(d, causal):
    lengths = [1, 17, 128, 129, 300, 700, 256, 255]
    inp = wl.draw(len(lengths), 8, 2, max(lengths), d, seed=1100 + d)
    check_against_padded(inp, lengths, causal=causal, scale=1 / np.sqrt(d),
                         what=f"d{d} causal{causal}")


def test_empty_sequence_in_the_pack():
    lengths = [40, 0, 300]
    inp = wl.draw(3, 4, 4, 300, 64, seed=1200)
    check_against_padded(inp, lengths, causal=True, scale=0.125, what="empty seq")


def test_bert_workload_packed():
    w = wl.BERT
    inp = wl.draw_workload(w)
    check_against_padded(inp, list(inp.seqlens), causal=False, scale=w.scale, what="bert packed")
