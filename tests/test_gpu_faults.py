"""Device-side failure detection of the weight-streaming GEMM, exercised without a GPU fault.

Every wait of the kernel on an mbarrier is bounded; when the limit runs out the kernel writes
W4_ERR_TIMEOUT to dev_status and returns, so the context stays usable.  The test drives that
path through the library's fault-injection export (not part of w4a16.h): the producer warps stop
after their first stage, so the compute warps wait for a stage that never arrives, with a 20 ms
limit.  A routed pair that names a token past the end of the activations is reported as
W4_ERR_INVALID_ARG (and read as token 0) instead of being loaded.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from oracle import moe
from w4a16_group_quantized_w4_b200 import _lib, api, synth
from tests._util import assert_rows_close, dev_bf16, dev_f32, dev_u32, host_f64

pytestmark = pytest.mark.gpu


def _stall_fn():
    lib = _lib.load()
    fn = lib.w4_testing_stream_gmm_stall
    fn.restype = C.c_int32
    P, I32, I64 = C.c_void_p, C.c_int32, C.c_int64
    fn.argtypes = [P, P, I32, P, P, P, I32, I64, I32, I32, I32, P, P, C.c_size_t, P, P,
                   C.c_uint64, I32]
    return fn


def test_stream_wait_runs_out_reports_timeout_and_next_call_is_correct():
    T, E, k, H, I = 4, 128, 8, 2816, 704          # decode-sized: the weight-streaming kernel
    case = synth.moe_case(T, E, k, H, I, seed=77)
    rt = api.moe_route_permute(dev_f32(case.logits), k)
    x, codes, scales = dev_bf16(case.x), dev_u32(case.gu_codes), dev_bf16(case.gu_scales)
    rows = T * k
    out = torch.zeros((rows, I), dtype=torch.bfloat16, device="cuda")
    need = api.w4_workspace_bytes(_lib.W4_OP_GMM, rows, 2 * I, H, E, k)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    rc = _stall_fn()(C.c_void_p(x.data_ptr()), C.c_void_p(rt.sorted_pair.data_ptr()), k,
                     C.c_void_p(codes.data_ptr()), C.c_void_p(scales.data_ptr()),
                     C.c_void_p(rt.expert_offsets.data_ptr()), E, rows, 2 * I, H,
                     _lib.W4_EPI_GELU_GATE, C.c_void_p(out.data_ptr()), C.c_void_p(ws.data_ptr()),
                     need, C.c_void_p(status.data_ptr()), C.c_void_p(stream.cuda_stream),
                     20_000_000, 1)
    assert rc == _lib.W4_OK
    torch.cuda.synchronize()
    assert status.item() == _lib.W4_ERR_TIMEOUT
    # the context is usable and the same stream computes the right answer next
    status.zero_()
    h = api.moe_w4a16_gmm(x, rt.sorted_pair, k, codes, scales, rt.expert_offsets, rows,
                          api.W4_EPI_GELU_GATE, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == _lib.W4_OK
    ref_rt = moe.route(case.logits, k)
    ref = moe.gmm(case.x, ref_rt.sorted_pair, k, case.gu_codes, case.gu_scales,
                  ref_rt.expert_offsets, moe.EPI_GELU_GATE)
    assert_rows_close(host_f64(h), ref)


def test_stream_bad_pair_index_reports_invalid_arg():
    """The weight-streaming kernel's preparation pass checks every routed pair against the rows of
    `a`: one naming a token past the end is reported and read as token 0; the other rows are
    right."""
    T, E, k, H, I = 16, 8, 2, 256, 128
    case = synth.moe_case(T, E, k, H, I, seed=19)
    rt = api.moe_route_permute(dev_f32(case.logits), k)
    bad = rt.sorted_pair.clone()
    bad_row = 5
    bad[bad_row] = T * k + 40
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = api.moe_w4a16_gmm(dev_bf16(case.x), bad, k, dev_u32(case.gu_codes), dev_bf16(case.gu_scales),
                            rt.expert_offsets, T * k, moe.EPI_GELU_GATE, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == _lib.W4_ERR_INVALID_ARG
    ref_rt = moe.route(case.logits, k)
    pairs = ref_rt.sorted_pair.copy()
    pairs[bad_row] = 0                              # read as token 0
    ref = moe.gmm(case.x, pairs, k, case.gu_codes, case.gu_scales, ref_rt.expert_offsets,
                  moe.EPI_GELU_GATE)
    assert_rows_close(host_f64(out), ref)
