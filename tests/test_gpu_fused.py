"""The fused single-launch MoE decode layer (moe_w4a16_layer) against the four-call path and the
oracle.

Pages: "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", sections
"What changed in vLLM's TPU backend" (the fused-MoE layer over packed int4 experts) and "The gap
at 26B" (128 experts, 8 active).  The fused kernel runs the arithmetic of moe_route_permute ->
moe_w4a16_gmm (gate/up, GELU gate) -> moe_w4a16_gmm (down) -> moe_combine on the weight-streaming
kernel in the same order, so its y must equal that path's y bit for bit; against the float64
oracle every token row meets the tolerance of the other GEMM tests (rel-L2 5e-3, max-abs
2e-2 * max|ref|).
"""
import numpy as np
import pytest
import torch

from oracle import moe
from w4a16_group_quantized_w4_b200 import _lib, api, synth
from tests._util import assert_rows_close, dev_bf16, dev_f32, dev_u32, host_bf16_bits, host_f64

pytestmark = pytest.mark.gpu


def _weights(case):
    return (dev_u32(case.gu_codes), dev_bf16(case.gu_scales), dev_u32(case.dn_codes),
            dev_bf16(case.dn_scales))


def _both(case, w=None):
    w = _weights(case) if w is None else w
    x, lg = dev_bf16(case.x), dev_f32(case.logits)
    y4 = api.MoELayer(*w, case.T, case.k)(x, lg).clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    yf = api.moe_w4a16_layer(x, lg, case.k, *w, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return host_bf16_bits(y4), host_bf16_bits(yf), yf


def _oracle(case, tokens=None):
    return moe.moe_layer(case.x, case.logits, case.gu_codes, case.gu_scales, case.dn_codes,
                         case.dn_scales, case.k, tokens=tokens)


@pytest.mark.parametrize("T", [1, 3, 64])
def test_fused_layer_full_config(T):
    """T decode tokens through 128 experts (top-8, hidden 2816, intermediate 704): one token
    splits the gate/up GEMM's K in three (the split-K reduction hands over through the counters
    too); 64 tokens reach nearly every expert."""
    case = synth.moe_case(T, 128, 8, 2816, 704, seed=300 + T)
    y4, yf, yt = _both(case)
    assert np.array_equal(yf, y4)
    assert_rows_close(host_f64(yt), _oracle(case).y)


@pytest.mark.parametrize("T,E,k,H,I,skew", [
    (1, 16, 4, 256, 128, None),
    (5, 8, 2, 64, 32, None),
    (20, 16, 4, 256, 96, None),        # T k = 80 of the 96 rows allowed: ragged blocks
    (48, 64, 8, 512, 160, None),       # T k = 6 E exactly; I / 64 ragged gate/up tiles
    (48, 64, 8, 512, 160, 1.1),        # Zipf-skewed experts: hot blocks and empty experts
    (10, 32, 16, 288, 64, None),       # k = 16 (combine in two batches); H ragged on 128
    (33, 8, 1, 128, 64, None),         # k = 1
])
def test_fused_layer_small_shapes(T, E, k, H, I, skew):
    case = synth.moe_case(T, E, k, H, I, seed=T * 7 + E + k, zipf_s=skew)
    y4, yf, yt = _both(case)
    assert np.array_equal(yf, y4)
    assert_rows_close(host_f64(yt), _oracle(case).y)


def test_fused_layer_ties():
    """Router logits with many exact ties (the lower expert index wins)."""
    case = synth.moe_case(12, 32, 4, 256, 64, seed=5)
    rng = np.random.default_rng(77)
    case.logits = rng.integers(-2, 3, size=(12, 32)).astype(np.float32)
    y4, yf, yt = _both(case)
    assert np.array_equal(yf, y4)
    assert_rows_close(host_f64(yt), _oracle(case).y)


def test_fused_layer_reuses_its_workspace():
    """One workspace, calls with 64, 1, 17 and 64 tokens back to back: each call starts from the
    zeroed control area the previous one left."""
    big = synth.moe_case(64, 128, 8, 2816, 704, seed=11)
    w = _weights(big)
    ws = api.layer_workspace(64, 128, 8, 2816, 704, "cuda")
    ctl = api.w4_workspace_bytes(_lib.W4_OP_LAYER_CTL, 0, 2816, 704, 128, 8)
    assert 0 < ctl < ws.numel()
    for T, seed in [(64, 1), (1, 2), (17, 3), (64, 4)]:
        case = synth.moe_case(T, 128, 8, 2816, 704, seed=seed)
        case.gu_codes, case.gu_scales, case.dn_codes, case.dn_scales = (
            big.gu_codes, big.gu_scales, big.dn_codes, big.dn_scales)
        x, lg = dev_bf16(case.x), dev_f32(case.logits)
        y4 = host_bf16_bits(api.MoELayer(*w, T, 8)(x, lg))
        yf = api.moe_w4a16_layer(x, lg, 8, *w, ws=ws)
        torch.cuda.synchronize()
        assert np.array_equal(host_bf16_bits(yf), y4)
        assert int(ws[:ctl].count_nonzero().item()) == 0


def test_fused_layer_in_cuda_graph():
    """The cooperative launch captured once and replayed with new inputs."""
    case = synth.moe_case(8, 128, 8, 2816, 704, seed=21)
    w = _weights(case)
    layer = api.MoELayer(*w, 8, 8, fused=True)
    x = dev_bf16(case.x)
    lg = dev_f32(case.logits)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer(x, lg)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        y = layer(x, lg)
    for seed in (22, 23):
        c2 = synth.moe_case(8, 128, 8, 2816, 704, seed=seed)
        x.copy_(dev_bf16(c2.x))
        lg.copy_(dev_f32(c2.logits))
        g.replay()
        torch.cuda.synchronize()
        y4 = host_bf16_bits(api.MoELayer(*w, 8, 8)(x, lg))
        torch.cuda.synchronize()
        assert np.array_equal(host_bf16_bits(y), y4)


def test_fused_layer_sizes_outside_its_range():
    w = _weights(synth.moe_case(1, 16, 4, 256, 128, seed=0))
    x = torch.zeros((129, 256), dtype=torch.bfloat16, device="cuda")
    lg = torch.zeros((129, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(_lib.W4Error) as ei:      # T > 128
        api.moe_w4a16_layer(x, lg, 4, *w, ws=torch.zeros(1 << 20, dtype=torch.uint8, device="cuda"))
    assert ei.value.status == _lib.W4_ERR_UNSUPPORTED
    x, lg = x[:25].contiguous(), lg[:25].contiguous()
    with pytest.raises(_lib.W4Error) as ei:      # T k = 100 > 6 E = 96
        api.moe_w4a16_layer(x, lg, 4, *w, ws=torch.zeros(1 << 20, dtype=torch.uint8, device="cuda"))
    assert ei.value.status == _lib.W4_ERR_UNSUPPORTED
