"""GPU parity of the weight-format variants (other group sizes along K, asymmetric zero-point)
against the oracle (oracle.variants).

Page: "What quantization really is", section "How the ruler works" (scale and optional
zero-point; asymmetric quantisation; group-wise granularity).  Tolerance per output row: rel-L2
<= 5e-3 and max-abs <= 2e-2 * max|ref|; the symmetric group-32 special case is compared bit for
bit with the main entry points.
"""
import numpy as np
import pytest
import torch

from oracle import moe, variants
from w4a16_group_quantized_w4_b200 import api, synth
from tests._util import assert_rows_close, dev_bf16, dev_f32, dev_u32, host_bf16_bits, host_f64

pytestmark = pytest.mark.gpu


def _asym_weights(N, K, group, seed):
    """Asymmetric quantisation (oracle) of shifted normal weights: groups not centred on zero."""
    rng = np.random.default_rng(seed)
    w = rng.normal(0.3, 1.0, size=(N, K)) * 0.02 + rng.normal(0, 0.01, size=(N, K // group)).repeat(group, 1)
    from oracle import bf16
    qz = variants.quantize_asym(bf16.from_f64(w), group)
    return qz.codes, qz.scales, qz.zeros


@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("zp", [False, True])
@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (4, 384, 2816), (16, 200, 1024), (33, 128, 4096)])
def test_linear_variants(group, zp, M, N, K):
    x = synth.bf16_normal((M, K), 0, 300 + M)
    if zp:
        codes, scales, zeros = _asym_weights(N, K, group, seed=M + group)
    else:
        codes = synth.random_code_words((N, K // 8), 0, 301)
        scales = synth.abs_normal_scales((N, K // group), 0.02, 1e-3, 0, 302)
        zeros = None
    y = api.w4a16_linear_g(dev_bf16(x), dev_u32(codes), dev_bf16(scales), group,
                           zeros=None if zeros is None else torch.from_numpy(zeros).cuda())
    torch.cuda.synchronize()
    ref = variants.linear(x, codes, scales, group, zeros)
    assert_rows_close(host_f64(y), ref)


def test_symmetric_group32_equals_main_entry_point():
    case = synth.dense_case(8, 512, 2816, 0.01, 1e-4, seed=17)
    x, c, s = dev_bf16(case.x), dev_u32(case.codes), dev_bf16(case.scales)
    y_main = api.w4a16_linear(x, c, s)
    y_var = api.w4a16_linear_g(x, c, s, 32)
    zeros8 = torch.full((case.N, case.K // 32), 8, dtype=torch.uint8, device="cuda")
    y_z8 = api.w4a16_linear_g(x, c, s, 32, zeros=zeros8)
    torch.cuda.synchronize()
    assert np.array_equal(host_bf16_bits(y_main), host_bf16_bits(y_var))
    assert_rows_close(host_f64(y_z8), host_f64(y_main).astype(np.float64))


@pytest.mark.parametrize("group", [64, 128])
@pytest.mark.parametrize("epi", [moe.EPI_NONE, moe.EPI_GELU_GATE])
def test_grouped_variants_with_zero_points(group, epi):
    T, E, k, H, I = 24, 16, 4, 512, 256
    logits = synth.router_logits(T, E, 0, 310)
    x = synth.bf16_normal((T, H), 0, 311)
    N = 2 * I if epi == moe.EPI_GELU_GATE else H
    codes = np.zeros((E, N, H // 8), np.uint32)
    scales = np.zeros((E, N, H // group), np.uint16)
    zeros = np.zeros((E, N, H // group), np.uint8)
    for e in range(E):
        codes[e], scales[e], zeros[e] = _asym_weights(N, H, group, seed=400 + e)
    rt = api.moe_route_permute(dev_f32(logits), k)
    out = api.moe_w4a16_gmm_g(dev_bf16(x), rt.sorted_pair, k, dev_u32(codes), dev_bf16(scales),
                              rt.expert_offsets, T * k, group, zeros=torch.from_numpy(zeros).cuda(),
                              epilogue=epi)
    torch.cuda.synchronize()
    ref_rt = moe.route(logits, k)
    ref = variants.gmm(x, ref_rt.sorted_pair, k, codes, scales, ref_rt.expert_offsets, epi, group, zeros)
    assert_rows_close(host_f64(out), ref)
