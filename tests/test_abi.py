"""The C ABI library: it loads, exports every entry point include/fa.h
declares, and rejects bad arguments synchronously (no GPU needed: argument
checks run before any CUDA call)."""
import os
import re

import pytest

from exact_io_aware_92_b200 import _lib
from exact_io_aware_92_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


def declared_entry_points():
    text = open(HEADER).read()
    return re.findall(r"FA_API\s+[\w\s\*]*?\b(fa_\w+)\s*\(", text)


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return _lib.load()


def test_header_declares_the_entry_points():
    names = declared_entry_points()
    assert "fa_fwd" in names and "fa_fwd_ex" in names and "fa_check_status" in names
    assert len(names) == len(set(names))


def test_library_exports_every_declared_symbol(lib):
    for name in declared_entry_points():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks a signature for {name}"


def test_status_strings(lib):
    for code in range(0, -11, -1):
        assert _lib.status_string(code) != "unknown status"
    assert _lib.status_string(-8) == "a bounded in-kernel wait ran out"
    assert _lib.status_string(12345) == "unknown status"
    assert lib.fa_version() == 100


A = 4096  # a 16-byte aligned fake address: never dereferenced, checks come first


@pytest.mark.parametrize("args,code", [
    ((None, A, A, A, A, 1, 2, 1, 128, 64, 0.125, 0, None), _lib.FA_ERR_NULL),
    ((A, A, A, A, None, 1, 2, 1, 128, 64, 0.125, 0, None), _lib.FA_ERR_NULL),
    ((A, A, A, A, A, 0, 2, 1, 128, 64, 0.125, 0, None), _lib.FA_ERR_SHAPE),
    ((A, A, A, A, A, 1, 2, 1, 0, 64, 0.125, 0, None), _lib.FA_ERR_SHAPE),
    ((A, A, A, A, A, 1, 2, 1, 128, 64, 0.0, 0, None), _lib.FA_ERR_SHAPE),
    ((A, A, A, A, A, 1, 2, 1, 128, 64, -1.0, 0, None), _lib.FA_ERR_SHAPE),
    ((A, A, A, A, A, 1, 2, 1, 128, 64, float("nan"), 0, None), _lib.FA_ERR_SHAPE),
    ((A, A, A, A, A, 1, 3, 2, 128, 64, 0.125, 0, None), _lib.FA_ERR_HEADS),
    ((A, A, A, A, A, 1, 2, 1, 128, 96, 0.125, 0, None), _lib.FA_ERR_HEADDIM),
    ((A, A, A, A, A, 1, 2, 1, 128, 32, 0.125, 0, None), _lib.FA_ERR_HEADDIM),
    ((A + 8, A, A, A, A, 1, 2, 1, 128, 64, 0.125, 0, None), _lib.FA_ERR_ALIGN),
    ((A, A, A, A + 2, A, 1, 2, 1, 128, 64, 0.125, 0, None), _lib.FA_ERR_ALIGN),
    ((A, A, A, A, A + 2, 1, 2, 1, 128, 64, 0.125, 0, None), _lib.FA_ERR_ALIGN),
])
def test_bad_arguments_rejected_before_launch(lib, args, code):
    assert lib.fa_fwd(*args) == code
    assert lib.fa_fwd_f32(*args) == code


def test_unknown_dtype_rejected(lib):
    rc = lib.fa_fwd_ex(A, A, A, A, A, 1, 2, 1, 128, 64, 0.125, 0, None, 7, None, None)
    assert rc == _lib.FA_ERR_DTYPE


def test_hostio_requires_device_seqlens_with_host_seqlens(lib):
    rc = lib.fa_fwd_hostio(A, A, A, A, A, A, A, A, A, A, A, None, 1, 2, 1, 128, 64, 0.125, 0, None)
    assert rc == _lib.FA_ERR_NULL


def test_hostio_async_rejects_bad_arguments_before_any_device_call(lib):
    # the asynchronous form validates exactly like the synchronous one
    rc = lib.fa_fwd_hostio_async(A, A, A, A, A, A, A, A, A, A, A, None, 1, 2, 1, 128, 64, 0.125, 0,
                                 None)
    assert rc == _lib.FA_ERR_NULL
    rc = lib.fa_fwd_hostio_async(None, A, A, A, A, None, A, A, A, A, A, None, 1, 2, 1, 128, 64,
                                 0.125, 0, None)
    assert rc == _lib.FA_ERR_NULL
    rc = lib.fa_fwd_hostio_async(A, A, A, A, A, None, A, A, A, A, A, None, 1, 3, 2, 128, 64, 0.125,
                                 0, None)
    assert rc == _lib.FA_ERR_HEADS
    rc = lib.fa_fwd_hostio_async(A, A, A, A, A, None, A, A, A, A, A, None, 1, 2, 1, 128, 96, 0.125,
                                 0, None)
    assert rc == _lib.FA_ERR_HEADDIM


def test_ex2_calibration_needs_an_output(lib):
    assert lib.fa_measure_ex2_rate(None, None) == _lib.FA_ERR_NULL


def test_decode_workspace_size_and_errors(lib):
    n = lib.fa_decode_workspace_size(8, 32, 8, 1, 32768, 128, 0)
    assert n > 0 and n % 4 == 0
    assert lib.fa_decode_workspace_size(8, 32, 8, 1, 32768, 96, 0) == 0  # bad head dim
    assert lib.fa_decode_workspace_size(8, 30, 8, 1, 32768, 128, 0) == 0  # Hq % Hkv
    more = lib.fa_decode_workspace_size(8, 32, 8, 1, 32768, 128, 64)
    assert more >= lib.fa_decode_workspace_size(8, 32, 8, 1, 32768, 128, 1)
    args = (A, A, A, A, A, 2, 8, 2, 1, 1000, 128, 0.088, 0)
    # missing or too-small workspace is reported before anything touches the device
    assert lib.fa_fwd_decode(*args, None, 0, None, 0, None, None) == _lib.FA_ERR_WORKSPACE
    assert lib.fa_fwd_decode(*args, None, 0, A, 16, None, None) == _lib.FA_ERR_WORKSPACE
    assert lib.fa_fwd_decode(*args, None, 0, A + 4, 1 << 30, None, None) == _lib.FA_ERR_WORKSPACE
    assert lib.fa_fwd_decode(*args, None, 200, A, 1 << 30, None, None) == _lib.FA_ERR_SHAPE
    assert lib.fa_fwd_decode(A, A, A, A, A, 2, 8, 3, 1, 1000, 128, 0.088, 0, None, 0, A, 1 << 30,
                             None, None) == _lib.FA_ERR_HEADS


def test_decode_workspace_sizes_of_both_kernels(lib):
    """Up to 128 query rows per kv head (G * Nq) take the tensor cores:
    partials for at most ctas + B * Hkv pieces, with ctas = 256 by default
    (one CTA per SM, at most 256) or min(num_splits * B * Hkv, 1024).  Each
    partial holds row slots of d + 2 floats: 16 up to 16 rows (keys on the
    tensor-memory lanes), the row count rounded up to 16 from 17 to 128 (rows
    on the lanes).  Beyond 128 rows the CUDA-core kernel's per-key-range
    partials apply."""
    def tc_bytes(B, Hkv, d, ctas, slots=16):
        pieces = ctas + B * Hkv
        o_bytes = pieces * slots * d * 4
        return (o_bytes + 255) // 256 * 256 + pieces * slots * 2 * 4

    assert lib.fa_decode_workspace_size(8, 32, 8, 1, 32768, 128, 0) == tc_bytes(8, 8, 128, 256)
    assert lib.fa_decode_workspace_size(8, 32, 8, 4, 32768, 64, 0) == tc_bytes(8, 8, 64, 256)
    assert lib.fa_decode_workspace_size(8, 32, 8, 8, 32768, 64, 0) == tc_bytes(8, 8, 64, 256, 32)
    assert lib.fa_decode_workspace_size(3, 8, 2, 1, 2000, 128, 7) == tc_bytes(3, 2, 128, 42)
    assert lib.fa_decode_workspace_size(64, 64, 16, 1, 4096, 128, 2) == tc_bytes(64, 16, 128, 1024)
    # 4 query heads per kv head: x 4 rows = 16 slots; x 5 = 20 rows -> 32 slots
    assert lib.fa_decode_workspace_size(2, 8, 2, 4, 1000, 128, 3) == tc_bytes(2, 2, 128, 12)
    assert lib.fa_decode_workspace_size(2, 8, 2, 5, 1000, 128, 3) == tc_bytes(2, 2, 128, 12, 32)
    # 8 x 16 = 128 rows: the last tensor-core shape; 8 x 17 = 136: CUDA cores
    assert lib.fa_decode_workspace_size(2, 8, 1, 16, 1000, 128, 3) == tc_bytes(2, 1, 128, 6, 128)
    cc = lib.fa_decode_workspace_size(2, 8, 1, 17, 1000, 128, 3)
    assert cc > 0 and cc != tc_bytes(2, 1, 128, 6, 144)


def test_without_a_b200_valid_calls_report_arch():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; covered by the gpu tests")
    lib = _lib.load()
    assert lib.fa_fwd(A, A, A, A, A, 1, 2, 1, 128, 64, 0.125, 0, None) == _lib.FA_ERR_ARCH
    assert lib.fa_check_status(None, None) == _lib.FA_ERR_ARCH


def test_fp8_arguments_rejected_before_launch(lib):
    # q, k, vt, o, lse, B, Hq, Hkv, N, ldvt, d, scale, descales, causal, seqlens, stream, status
    def call(N=300, ldvt=304, d=128, dq=0.01, dk=0.01, dv=0.01, Hq=8, Hkv=2, q=A):
        return lib.fa_fwd_fp8(q, A, A, A, A, 2, Hq, Hkv, N, ldvt, d, 0.088, dq, dk, dv, 1, None,
                              None, None)
    assert call(d=64) == _lib.FA_ERR_HEADDIM          # FP8 path: head dim 128 only
    assert call(ldvt=296) == _lib.FA_ERR_SHAPE         # ldvt < N
    assert call(ldvt=312 - 4) == _lib.FA_ERR_ALIGN     # not a multiple of 16
    assert call(dq=0.0) == _lib.FA_ERR_SHAPE
    assert call(dv=float("inf")) == _lib.FA_ERR_SHAPE
    assert call(Hq=6, Hkv=4) == _lib.FA_ERR_HEADS
    assert call(q=None) == _lib.FA_ERR_NULL
    assert call(q=A + 8) == _lib.FA_ERR_ALIGN
