"""fa_fwd_decode_noalloc: decode for callers that cannot allocate device
memory (a fixed-budget inference loop, a host framework that owns every
allocation, a latency path that cannot afford cudaMalloc's implicit device
synchronisation).  It keeps its partials in the library's own 8 MiB device
array instead of a caller workspace.

The test calls it through the C ABI twice in a row, on different inputs, and
checks each result against fa_fwd_decode with a caller-provided workspace,
within the tolerances the parity tests use.  It creates everything it needs,
so it passes alone in a fresh process as well as after the other tests.
"""
import numpy as np
import pytest

from exact_io_aware_92_b200 import _lib
from exact_io_aware_92_b200 import workloads as wl
from parity_helpers import LSE_TOL_BF16, O_TOL_BF16, compare, to_device_bf16

pytestmark = pytest.mark.gpu


def _call(fn_name, inp, B, Hq, Hkv, Nq, Nk, d, *, causal, scale, workspace=None):
    import torch
    lib = _lib.load()
    q, k, v = (to_device_bf16(x) for x in (inp.q_bits, inp.k_bits, inp.v_bits))
    sl = None if inp.seqlens is None else torch.from_numpy(inp.seqlens).cuda()
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    common = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
              B, Hq, Hkv, Nq, Nk, d, scale, int(causal), None if sl is None else sl.data_ptr(), 0)
    if fn_name == "fa_fwd_decode_noalloc":
        rc = lib.fa_fwd_decode_noalloc(*common, stream, status.data_ptr())
    else:
        rc = lib.fa_fwd_decode(*common, workspace.data_ptr(), workspace.numel(), stream,
                               status.data_ptr())
    assert rc == _lib.FA_OK, _lib.status_string(rc)
    assert lib.fa_check_status(status.data_ptr(), stream) == _lib.FA_OK
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("call", [0, 1])
def test_noalloc_matches_workspace_entry_point_on_two_calls(call):
    import torch
    lib = _lib.load()
    # two different shapes and inputs, run back to back through the shared array
    cases = [
        dict(B=4, Hq=32, Hkv=8, Nq=1, Nk=8192, d=128, causal=True, seed=901, lens=None),
        dict(B=3, Hq=16, Hkv=4, Nq=2, Nk=3000, d=64, causal=True, seed=902, lens=[3000, 1, 1500]),
    ]
    outs = []
    for c in cases:
        inp = wl.draw(c["B"], c["Hq"], c["Hkv"], c["Nk"], c["d"], c["seed"], nq=c["Nq"])
        if c["lens"] is not None:
            inp.seqlens = np.array(c["lens"], dtype=np.int32)
        shape = (c["B"], c["Hq"], c["Hkv"], c["Nq"], c["Nk"], c["d"])
        scale = 1.0 / np.sqrt(c["d"])
        need = lib.fa_decode_workspace_size(*shape, 0)
        assert 0 < need <= 8 << 20
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        ref = _call("fa_fwd_decode", inp, *shape, causal=c["causal"], scale=scale, workspace=ws)
        got = _call("fa_fwd_decode_noalloc", inp, *shape, causal=c["causal"], scale=scale)
        outs.append((got, ref))
    for (o, lse), (o_r, l_r) in outs:
        compare(o, lse, o_r, l_r, o_tol=O_TOL_BF16, lse_tol=LSE_TOL_BF16, what=f"call {call}")


def test_noalloc_rejects_shapes_beyond_its_array():
    lib = _lib.load()
    A = 4096  # never dereferenced: the size check comes first
    # 64 key ranges x 2048 query rows x (128 + 2) floats is far beyond 8 MiB
    rc = lib.fa_fwd_decode_noalloc(A, A, A, A, A, 8, 32, 8, 8, 32768, 128, 0.088, 1, None, 64,
                                   None, None)
    assert rc == _lib.FA_ERR_WORKSPACE
