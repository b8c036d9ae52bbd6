"""fa_fwd_decode_noalloc: decode for callers that cannot allocate device
memory (a fixed-budget inference loop, a host framework that owns every
allocation, a latency path that cannot afford cudaMalloc's implicit device
synchronisation).  It keeps its partials in the library's own 8 MiB device
array instead of a caller workspace.

The test queues three calls in a row through the C ABI on one stream, the
largest layout first, so that each later call runs over the partials an
earlier one left in the shared array.  Only then are the outputs read, and
each is checked element by element against the fp64 oracle (queries at the
end of their sequences) within the tolerances of the parity tests, and
against fa_fwd_decode with a caller-provided workspace on the same inputs.
It creates everything it needs, so it passes alone in a fresh process as
well as after the other tests.
"""
import numpy as np
import pytest

import oracle
from exact_io_aware_92_b200 import _lib
from exact_io_aware_92_b200 import workloads as wl
from parity_helpers import LSE_TOL_BF16, O_TOL_BF16, compare, to_device_bf16

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 8 << 20

# Largest layout first, so that each later call runs over partials that an
# earlier, larger one left in the shared array: 32 rows per kv head (the
# rows-on-lanes kernel), then 4 and 8 (keys on the lanes).
CASES = [
    dict(B=2, Hq=16, Hkv=2, Nq=4, Nk=6000, d=128, causal=True, seed=903, lens=[6000, 2500]),
    dict(B=4, Hq=32, Hkv=8, Nq=1, Nk=8192, d=128, causal=True, seed=901, lens=None),
    dict(B=3, Hq=16, Hkv=4, Nq=2, Nk=3000, d=64, causal=True, seed=902, lens=[3000, 1, 1500]),
]


def _prepare(c):
    import torch
    inp = wl.draw(c["B"], c["Hq"], c["Hkv"], c["Nk"], c["d"], c["seed"], nq=c["Nq"])
    if c["lens"] is not None:
        inp.seqlens = np.array(c["lens"], dtype=np.int32)
    t = dict(inp=inp, shape=(c["B"], c["Hq"], c["Hkv"], c["Nq"], c["Nk"], c["d"]),
             scale=1.0 / np.sqrt(c["d"]), causal=c["causal"])
    t["q"], t["k"], t["v"] = (to_device_bf16(x) for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    t["sl"] = None if inp.seqlens is None else torch.from_numpy(inp.seqlens).cuda()
    return t


def _outputs(t):
    import torch
    B, Hq, _, Nq, _, _ = t["shape"]
    return torch.empty_like(t["q"]), torch.empty((B, Hq, Nq), dtype=torch.float32, device="cuda")


def _args(t, o, lse):
    return (t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), o.data_ptr(),
            lse.data_ptr(), *t["shape"], t["scale"], int(t["causal"]),
            None if t["sl"] is None else t["sl"].data_ptr(), 0)


def _host(o, lse):
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def test_noalloc_calls_in_a_row_match_oracle_and_workspace_entry_point():
    import torch
    lib = _lib.load()
    stream = torch.cuda.current_stream().cuda_stream
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cases = [_prepare(c) for c in CASES]
    # the no-allocation calls queued back to back, nothing read in between
    got = []
    for t in cases:
        assert 0 < lib.fa_decode_workspace_size(*t["shape"], 0) <= SCRATCH_BYTES
        o, lse = _outputs(t)
        rc = lib.fa_fwd_decode_noalloc(*_args(t, o, lse), stream, status.data_ptr())
        assert rc == _lib.FA_OK, _lib.status_string(rc)
        got.append((o, lse))
    assert lib.fa_check_status(status.data_ptr(), stream) == _lib.FA_OK
    for t, (o_d, lse_d) in zip(cases, got):
        o, lse = _host(o_d, lse_d)
        inp = t["inp"]
        what = "B{} Hq{} Hkv{} Nq{} Nk{} d{}".format(*t["shape"])
        o_ref, lse_ref = oracle.attention_forward(
            inp.q_bits, inp.k_bits, inp.v_bits, causal=t["causal"],
            scale=float(np.float32(t["scale"])), seqlens=inp.seqlens, causal_bottom_right=True)
        compare(o, lse, o_ref, lse_ref, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16,
                what=f"no-alloc vs oracle, {what}")
        ws = torch.empty(lib.fa_decode_workspace_size(*t["shape"], 0), dtype=torch.uint8,
                         device="cuda")
        o_w, lse_w = _outputs(t)
        rc = lib.fa_fwd_decode(*_args(t, o_w, lse_w), ws.data_ptr(), ws.numel(), stream,
                               status.data_ptr())
        assert rc == _lib.FA_OK, _lib.status_string(rc)
        assert lib.fa_check_status(status.data_ptr(), stream) == _lib.FA_OK
        o_r, lse_r = _host(o_w, lse_w)
        compare(o, lse, o_r, lse_r, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16,
                what=f"no-alloc vs workspace entry point, {what}")


def test_noalloc_rejects_shapes_beyond_its_array():
    # Real device buffers of the stated shape: 512 query rows per kv head
    # with 64 key ranges need 16.8 MB of partials, twice the array, so the
    # call must be refused before anything is launched.
    import torch
    lib = _lib.load()
    B, Hq, Hkv, Nq, Nk, d, splits = 1, 64, 1, 8, 16384, 128, 64
    need = lib.fa_decode_workspace_size(B, Hq, Hkv, Nq, Nk, d, splits)
    assert need > SCRATCH_BYTES
    q = torch.zeros((B, Hq, Nq, d), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((B, Hkv, Nk, d), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.fa_fwd_decode_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   lse.data_ptr(), B, Hq, Hkv, Nq, Nk, d, 0.088, 1, None, splits,
                                   stream, status.data_ptr())
    assert rc == _lib.FA_ERR_WORKSPACE
    assert lib.fa_check_status(status.data_ptr(), stream) == _lib.FA_OK
