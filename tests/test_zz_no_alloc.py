"""The allocation-free dense linear (w4a16_linear_noalloc) agrees with w4a16_linear.

Some callers are handed only input and output buffers and may not allocate device memory (a
plugin inside a framework that owns every device byte through its own pool, or a runtime held to
a fixed budget).  w4a16_linear_noalloc serves them from the library's fixed 8 MiB device array
instead of a caller workspace.  This test calls it through the C ABI twice in a row and checks
both results against the regular entry point, within the tolerance the other GEMM tests use.
It lives in a file of its own that pytest collects last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from w4a16_group_quantized_w4_b200 import _lib, api, synth
from tests._util import assert_rows_close, dev_bf16, dev_u32, host_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M", [1, 4, 16])
def test_noalloc_matches_workspace_entry_point(M):
    lib = _lib.load()
    case = synth.case_dense_gemv(M, seed=7)
    x, codes, scales = dev_bf16(case.x), dev_u32(case.codes), dev_bf16(case.scales)
    need = api.w4_workspace_bytes(_lib.W4_OP_LINEAR, M, case.N, case.K, 1, 1)
    assert 0 < need <= api.NOALLOC_SCRATCH_BYTES          # the split-K path (uses scratch) runs
    ref = host_f64(api.w4a16_linear(x, codes, scales))
    for _ in range(2):                                    # two calls in a row share the scratch
        y = torch.full((M, case.N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = C.c_void_p(torch.cuda.current_stream().cuda_stream)
        status = lib.w4a16_linear_noalloc(C.c_void_p(x.data_ptr()), C.c_void_p(codes.data_ptr()),
                                          C.c_void_p(scales.data_ptr()), C.c_void_p(y.data_ptr()),
                                          M, case.N, case.K, st)
        assert status == _lib.W4_OK, lib.w4_status_str(status)
        torch.cuda.synchronize()
        assert_rows_close(host_f64(y), ref)


def test_noalloc_splits_rows_that_do_not_fit_its_scratch():
    """63 rows against K = 65536: the prepared activation rows alone (fp16 values, corrections
    and multipliers of every 16-row block) exceed the 8 MiB array, so the call runs the rows in
    chunks; the result must match the regular entry point."""
    lib = _lib.load()
    M, N, K = 63, 256, 65536
    need = api.w4_workspace_bytes(_lib.W4_OP_LINEAR, M, N, K, 1, 1)
    assert need > api.NOALLOC_SCRATCH_BYTES
    case = synth.dense_case(M, N, K, 0.01, 1e-4, seed=11)
    x, codes, scales = dev_bf16(case.x), dev_u32(case.codes), dev_bf16(case.scales)
    ref = host_f64(api.w4a16_linear(x, codes, scales))
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    status = lib.w4a16_linear_noalloc(C.c_void_p(x.data_ptr()), C.c_void_p(codes.data_ptr()),
                                      C.c_void_p(scales.data_ptr()), C.c_void_p(y.data_ptr()),
                                      M, N, K, st)
    assert status == _lib.W4_OK, lib.w4_status_str(status)
    torch.cuda.synchronize()
    assert_rows_close(host_f64(y), ref)


def test_noalloc_rejects_a_row_beyond_its_scratch():
    lib = _lib.load()
    # K = 2^22: one prepared row is 10 MiB, over the fixed 8 MiB, so the call must refuse before
    # launching anything (the dummy buffers are never touched)
    M, N, K = 1, 8, 1 << 22
    need = api.w4_workspace_bytes(_lib.W4_OP_LINEAR, M, N, K, 1, 1)
    assert need > api.NOALLOC_SCRATCH_BYTES
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = C.c_void_p(dummy.data_ptr())
    status = lib.w4a16_linear_noalloc(p, p, p, p, M, N, K, C.c_void_p(None))
    assert status == _lib.W4_ERR_WORKSPACE


def test_noalloc_last_chunk_that_needs_more_scratch_than_the_others():
    """289 rows against N = 2048, K = 16384: the rows run in chunks, and the shorter last chunk
    makes fewer work units, so it can split K and need float32 partials that the longer chunks
    do not.  The call must size its chunks so that every launch fits the 8 MiB array and match
    the regular entry point on every row."""
    lib = _lib.load()
    M, N, K = 289, 2048, 16384
    case = synth.dense_case(M, N, K, 0.01, 1e-4, seed=13)
    x, codes, scales = dev_bf16(case.x), dev_u32(case.codes), dev_bf16(case.scales)
    ref = host_f64(api.w4a16_linear(x, codes, scales))
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = C.c_void_p(torch.cuda.current_stream().cuda_stream)
        status = lib.w4a16_linear_noalloc(C.c_void_p(x.data_ptr()), C.c_void_p(codes.data_ptr()),
                                          C.c_void_p(scales.data_ptr()), C.c_void_p(y.data_ptr()),
                                          M, N, K, st)
        assert status == _lib.W4_OK, lib.w4_status_str(status)
        torch.cuda.synchronize()
        assert_rows_close(host_f64(y), ref)
