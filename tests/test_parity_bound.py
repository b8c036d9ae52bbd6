"""The per-element O bound of the bf16 stress test (parity_helpers.derived_o_bound),
checked on the CPU against emulations of the kernel's arithmetic.

The emulation rounds every probability to bf16 before the P.V product,
normalises by the fp32 sum of the unrounded probabilities and rounds O to
bf16, as the kernel does.  It must stay inside the bound.  An emulation that
keeps only 4 significant bits of P (a plausible mistake in the packing: a
wrong conversion) must break it, so the bound is not vacuous."""
import numpy as np
import torch

from exact_io_aware_92_b200 import workloads as wl
from parity_helpers import compare, derived_o_bound, reference

SCALE = 1.0 / np.sqrt(128)


def _emulate(p, inp, group, p_bits):
    pt = torch.from_numpy(p)
    if p_bits == 8:
        pr = pt.to(torch.bfloat16).double()
    else:  # keep p_bits significant bits
        m, e = torch.frexp(pt)
        pr = torch.ldexp(torch.round(m * 2 ** p_bits) / 2 ** p_bits, e)
    v = torch.from_numpy(wl.bf16_bits_to_f32(inp.v_bits)).double().repeat_interleave(group, dim=1)
    o = (pr @ v) / pt.float().double().sum(-1, keepdim=True)
    return o.to(torch.bfloat16).double().numpy()


def _case():
    inp = wl.draw(1, 4, 2, 700, 128, 5, k_scale=8.0)
    o_ref, lse_ref, p = reference(inp, causal=True, scale=SCALE, return_probs=True)
    return inp, o_ref, lse_ref, p, derived_o_bound(inp, p, o_ref, float(np.float32(SCALE)))


def test_kernel_rounding_stays_inside_the_bound():
    inp, o_ref, lse_ref, p, bound = _case()
    o = _emulate(p, inp, 2, 8)
    _, _, n_over = compare(o, lse_ref, o_ref, lse_ref, o_tol=1.5e-2, lse_tol=2e-3, o_bound=bound)
    assert float((np.abs(o - o_ref) / bound).max()) < 1.0
    assert n_over <= 36


def test_coarser_probabilities_break_the_bound():
    inp, o_ref, lse_ref, p, bound = _case()
    o = _emulate(p, inp, 2, 4)
    assert float((np.abs(o - o_ref) / bound).max()) > 1.0


def _bwd_emulation(inp, dout_bits, p, o_ref, scale, p_bits=8):
    """The backward's roundings on exact values: bf16 P for dV, D from the
    bf16 O, dS rounded to bf16 (or to p_bits bits), gradients rounded to bf16."""
    def rnd(x, bits):
        t = torch.from_numpy(x)
        if bits == 8:
            return t.to(torch.bfloat16).double().numpy()
        m, e = torch.frexp(t)
        return torch.ldexp(torch.round(m * 2 ** bits) / 2 ** bits, e).numpy()
    q, k, v, do = (wl.bf16_bits_to_f32(x).astype(np.float64)
                   for x in (inp.q_bits, inp.k_bits, inp.v_bits, dout_bits))
    G = q.shape[1] // k.shape[1]
    o16 = rnd(o_ref, 8)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            g = h // G
            P = p[b, h]
            D = (do[b, h] * o16[b, h]).sum(axis=1)
            dS = rnd(P * (do[b, h] @ v[b, g].T - D[:, None]), p_bits)
            dv[b, g] += rnd(P, p_bits).T @ do[b, h]
            dk[b, g] += scale * dS.T @ q[b, h]
            dq[b, h] = scale * dS @ k[b, g]
    return tuple(rnd(x, 8) for x in (dq, dk, dv))


def _bwd_case(p_bits):
    import oracle
    from parity_helpers import derived_grad_bounds
    scale = float(np.float32(1.0 / np.sqrt(64)))
    inp = wl.draw(1, 4, 2, 200, 64, 1300, k_scale=2.0)
    dout_bits = wl.round_to_bf16_bits(
        np.random.default_rng(7).standard_normal((1, 4, 200, 64), dtype=np.float32))
    o_ref, lse_ref, p = reference(inp, causal=True, scale=1.0 / np.sqrt(64), return_probs=True)
    ref = oracle.attention_backward(inp.q_bits, inp.k_bits, inp.v_bits, dout_bits, causal=True,
                                    scale=scale)
    o_bound = derived_o_bound(inp, p, o_ref, scale)
    bounds = derived_grad_bounds(inp, dout_bits, p, o_ref, o_bound, ref, scale)
    em = _bwd_emulation(inp, dout_bits, p, o_ref, scale, p_bits)
    return [float((np.abs(g - r) / bd).max()) for g, r, bd in zip(em, ref, bounds)]


def test_backward_rounding_stays_inside_the_gradient_bound():
    assert max(_bwd_case(8)) < 1.0


def test_coarser_backward_operands_break_the_gradient_bound():
    assert max(_bwd_case(4)) > 1.0
