"""GPU parity of the tensor-core (tcgen05) path against the float64 oracle.

Definition: "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", section
"What changed in vLLM's TPU backend": a scale per 32-wide group, each weight tile dequantised in
on-chip memory before the multiply, bf16 activations.  Shapes here are ones the library sends to
the tensor-core kernel (dense: M >= 64 and N % 128 == 0; grouped: on average >= 32 routed rows per
expert), which is checked through the workspace it asks for.  Tolerance per output row: rel-L2
<= 5e-3 and max-abs <= 2e-2 * max|y_ref|.
"""
import numpy as np
import pytest
import torch

from oracle import linear, moe, q4
from w4a16_group_quantized_w4_b200 import _lib, api, synth
from tests._util import assert_rows_close, dev_bf16, dev_f32, dev_u32, host_f64

pytestmark = pytest.mark.gpu


def _tc_bytes(rows, K, wrows):
    """fp16 rows and row multipliers (each 256-byte aligned), then one exponent byte per weight row."""
    return (rows * K * 2 + 255) // 256 * 256 + (rows * 4 + 255) // 256 * 256 + wrows


@pytest.mark.parametrize("M,N,K", [(64, 128, 64), (128, 128, 256), (200, 384, 512),
                                   (513, 128, 2816), (130, 256, 4096), (1000, 1408 * 2, 704)])
def test_dense_tc_shapes(M, N, K):
    assert api.w4_workspace_bytes(_lib.W4_OP_LINEAR, M, N, K, 1, 1) == _tc_bytes(M, K, N)
    case = synth.dense_case(M, N, K, 0.02, 1e-3, seed=M + 3 * N + K)
    y = api.w4a16_linear(dev_bf16(case.x), dev_u32(case.codes), dev_bf16(case.scales))
    torch.cuda.synchronize()
    assert_rows_close(host_f64(y), linear.w4a16_linear(case.x, case.codes, case.scales))


def test_dense_tc_wide_dynamic_range():
    """Activation rows from 1e-20 to 1e19 (far outside fp16) and scales spanning 2^-20 .. 2^10
    inside one weight row: the power-of-two row and column exponents keep every product exact."""
    M, N, K = 160, 256, 1024
    rng = np.random.default_rng(61)
    x = rng.standard_normal((M, K)) * (10.0 ** (np.arange(M) % 40 - 20))[:, None]
    s = 2.0 ** rng.uniform(-20, 10, size=(N, K // 32))
    q = rng.integers(-8, 8, size=(N, K))
    x_bits = synth.f32_to_bf16_bits(x.astype(np.float32))
    s_bits = synth.f32_to_bf16_bits(s.astype(np.float32))
    codes = q4.pack(q)
    y = api.w4a16_linear(dev_bf16(x_bits), dev_u32(codes), dev_bf16(s_bits))
    torch.cuda.synchronize()
    assert_rows_close(host_f64(y), linear.w4a16_linear(x_bits, codes, s_bits))


def test_dense_tc_small_workspace_is_an_error():
    M, N, K = 128, 128, 256
    case = synth.dense_case(M, N, K, 0.02, 1e-3, seed=5)
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(_lib.W4Error) as e:
        api.w4a16_linear(dev_bf16(case.x), dev_u32(case.codes), dev_bf16(case.scales), ws=ws)
    assert e.value.status == _lib.W4_ERR_WORKSPACE


def _route(logits, k):
    return api.moe_route_permute(dev_f32(logits), k)


@pytest.mark.parametrize("T,E,k,H,I,zipf", [(512, 8, 2, 256, 128, None), (1024, 16, 4, 512, 256, 1.5),
                                            (300, 4, 2, 128, 64, None)])
def test_grouped_tc_gate_up_and_down(T, E, k, H, I, zipf):
    case = synth.moe_case(T, E, k, H, I, seed=T + E, zipf_s=zipf)
    assert api.w4_workspace_bytes(_lib.W4_OP_GMM, T * k, 2 * I, H, E, k) == _tc_bytes(T * k, H, E * 2 * I)
    rt = _route(case.logits, k)
    ref_rt = moe.route(case.logits, k)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    h = api.moe_w4a16_gmm(dev_bf16(case.x), rt.sorted_pair, k, dev_u32(case.gu_codes),
                          dev_bf16(case.gu_scales), rt.expert_offsets, T * k, moe.EPI_GELU_GATE,
                          dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref_h = moe.gmm(case.x, ref_rt.sorted_pair, k, case.gu_codes, case.gu_scales,
                    ref_rt.expert_offsets, moe.EPI_GELU_GATE)
    assert_rows_close(host_f64(h), ref_h, what="h")
    # down projection on the device's own h (contiguous rows, no epilogue)
    h_bits = h.cpu().view(torch.int16).numpy().view(np.uint16)
    o = api.moe_w4a16_gmm(h, None, 1, dev_u32(case.dn_codes), dev_bf16(case.dn_scales),
                          rt.expert_offsets, T * k, moe.EPI_NONE, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref_o = moe.gmm(h_bits, None, 1, case.dn_codes, case.dn_scales, ref_rt.expert_offsets,
                    moe.EPI_NONE)
    assert_rows_close(host_f64(o), ref_o, what="o")


def test_grouped_tc_bad_pair_index_reports_invalid_arg():
    """A routed pair naming a token past the end of `a` is reported in dev_status (and read as
    token 0) instead of being loaded."""
    T, E, k, H, I = 256, 4, 2, 128, 64
    case = synth.moe_case(T, E, k, H, I, seed=9)
    rt = _route(case.logits, k)
    bad = rt.sorted_pair.clone()
    bad[7] = T * k + 40
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.moe_w4a16_gmm(dev_bf16(case.x), bad, k, dev_u32(case.gu_codes), dev_bf16(case.gu_scales),
                      rt.expert_offsets, T * k, moe.EPI_GELU_GATE, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == _lib.W4_ERR_INVALID_ARG
