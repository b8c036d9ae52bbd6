"""Attention backward (fa_bwd) vs the fp64 backward oracle on the same bf16
inputs.  The GPU forward supplies O and LSE, as in training.

Tolerance (no figure is stated for the backward; derived from the
arithmetic): each gradient element is a sum of products in which the
probabilities P (for dV) and dS = P (dP - D) (for dK, dQ) enter the tensor
cores rounded to bf16 (unit roundoff 2^-8), D comes from the bf16 forward
output, and the result is rounded to bf16 (2^-9 relative).  With independent
rounding errors over the summed terms, the error of each tensor stays a small
fraction of its largest element; the test requires
    max |g - g_ref| <= 1e-2 * max |g_ref| + 1e-3
for each of dQ, dK, dV, and reports the errors it saw."""
import numpy as np
import pytest

from exact_io_aware_92_b200 import workloads as wl
from parity_helpers import to_device_bf16

pytestmark = pytest.mark.gpu

import oracle  # noqa: E402

REL = 1e-2
ABS = 1e-3


def run_case(B, Hq, Hkv, N, d, causal, seed, seqlens=None):
    import torch
    from exact_io_aware_92_b200 import attention
    inp = wl.draw(B, Hq, Hkv, N, d, seed)
    dout_bits = wl.round_to_bf16_bits(
        np.random.default_rng(seed + 7).standard_normal((B, Hq, N, d), dtype=np.float32))
    q, k, v, do = (to_device_bf16(x) for x in (inp.q_bits, inp.k_bits, inp.v_bits, dout_bits))
    sl = None if seqlens is None else torch.from_numpy(np.asarray(seqlens, np.int32)).cuda()
    scale = 1.0 / np.sqrt(d)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = attention.fwd(q, k, v, causal=causal, scale=scale, seqlens=sl, status=status)
    dq, dk, dv = attention.bwd(q, k, v, o, do, lse, causal=causal, scale=scale, seqlens=sl,
                               status=status)
    assert attention.check_status(status) == 0
    ref = oracle.attention_backward(inp.q_bits, inp.k_bits, inp.v_bits, dout_bits, causal=causal,
                                    scale=float(np.float32(scale)),
                                    seqlens=None if seqlens is None else np.asarray(seqlens))
    out = {}
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        g = g.float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(g)), name
        err = float(np.abs(g - r).max())
        bound = REL * float(np.abs(r).max()) + ABS
        out[name] = (err, float(np.abs(r).max()))
        assert err <= bound, f"{name}: max|d| {err:.3e} > {bound:.3e} (max|ref| {np.abs(r).max():.3e})"
    return out


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 128, 200, 513])
def test_backward_shapes(N, d, causal):
    print(run_case(1, 2, 1, N, d, causal, seed=1300 + N))


@pytest.mark.parametrize("group", [1, 4])
def test_backward_gqa_and_padding(group):
    print(run_case(3, 8, 8 // group, 300, 128, True, seed=1400 + group, seqlens=[300, 0, 150]))
    print(run_case(2, 4, 4 // min(group, 4), 260, 64, False, seed=1410 + group, seqlens=[1, 260]))


def test_backward_llama_layer_shape():
    # one layer's worth of the GQA workload at N = 1024 (the oracle's fp64
    # backward of the full N = 8192 layer would take hours on the host)
    print(run_case(1, 8, 2, 1024, 128, True, seed=1500))
