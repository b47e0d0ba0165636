"""GPU parity of the MoE entry points against the oracle.

Pages: "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", sections
"The gap at 26B" (128 experts per layer, 8 active per token) and "What changed in vLLM's TPU
backend" (grouped matmul over packed int4 experts with per-32 scales, bf16 activations).
Routing ids, offsets and permutations are compared bit for bit; weights within 1e-6 relative;
GEMM outputs per row within rel-L2 5e-3 and max-abs 2e-2 * max|ref|.
"""
import numpy as np
import pytest
import torch

from oracle import bf16, moe
from w4a16_group_quantized_w4_b200 import _lib, api, synth
from tests._util import assert_rows_close, dev_bf16, dev_f32, dev_u32, host_f64

pytestmark = pytest.mark.gpu


def _route(logits, k):
    rt = api.moe_route_permute(dev_f32(logits), k)
    torch.cuda.synchronize()
    return rt


def _check_route(logits, k):
    ref = moe.route(logits, k)
    rt = _route(logits, k)
    assert np.array_equal(rt.topk_ids.cpu().numpy(), ref.topk_ids)
    assert np.array_equal(rt.expert_offsets.cpu().numpy(), ref.expert_offsets)
    assert np.array_equal(rt.sorted_pair.cpu().numpy(), ref.sorted_pair)
    assert np.array_equal(rt.pair_pos.cpu().numpy(), ref.pair_pos)
    w = rt.topk_w.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(w - ref.topk_w) <= 1e-6 * np.abs(ref.topk_w))
    return ref, rt


@pytest.mark.parametrize("T,E,k", [(1, 128, 8), (7, 128, 8), (64, 128, 8), (256, 128, 8),
                                   (257, 128, 8), (1000, 128, 8), (300, 8, 2), (50, 1024, 32),
                                   (33, 5, 1), (40, 16, 16)])
def test_route_permute(T, E, k):
    _check_route(synth.router_logits(T, E, 0, T + E), k)


def test_route_ties_and_zipf():
    rng = np.random.default_rng(41)
    ties = rng.integers(-2, 3, size=(600, 128)).astype(np.float32)
    _check_route(ties, 8)
    _check_route(synth.router_logits(8192, 128, 0, 102, zipf_s=synth.ZIPF_S), 8)


def test_route_empty():
    rt = api.moe_route_permute(torch.empty((0, 128), dtype=torch.float32, device="cuda"), 8)
    torch.cuda.synchronize()
    assert (rt.expert_offsets.cpu() == 0).all()


def _small_moe(T, E, k, H, I, seed, skew=None):
    return synth.moe_case(T, E, k, H, I, seed=seed, zipf_s=skew)


@pytest.mark.parametrize("epi", [moe.EPI_NONE, moe.EPI_GELU_GATE])
@pytest.mark.parametrize("T,E,k,H,I", [(5, 8, 2, 64, 32), (64, 16, 4, 256, 96),
                                       (300, 8, 2, 96, 160), (1, 128, 8, 256, 64)])
def test_gmm_gathered(epi, T, E, k, H, I):
    case = _small_moe(T, E, k, H, I, seed=T + E)
    rt = _route(case.logits, k)
    ref_rt = moe.route(case.logits, k)
    out = api.moe_w4a16_gmm(dev_bf16(case.x), rt.sorted_pair, k, dev_u32(case.gu_codes),
                            dev_bf16(case.gu_scales), rt.expert_offsets, T * k, epi)
    torch.cuda.synchronize()
    ref = moe.gmm(case.x, ref_rt.sorted_pair, k, case.gu_codes, case.gu_scales,
                  ref_rt.expert_offsets, epi)
    assert_rows_close(host_f64(out), ref)


def test_gmm_contiguous_rows_with_empty_and_hot_experts():
    rng = np.random.default_rng(43)
    E, N, K = 6, 136, 192
    counts = np.array([0, 70, 1, 0, 33, 5])
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(offs[-1])
    a = synth.bf16_normal((rows, K), 0, 44)
    codes = synth.random_code_words((E, N, K // 8), 0, 45)
    scales = synth.abs_normal_scales((E, N, K // 32), 0.02, 1e-3, 0, 46)
    out = api.moe_w4a16_gmm(dev_bf16(a), None, 1, dev_u32(codes), dev_bf16(scales),
                            torch.from_numpy(offs).cuda(), rows, moe.EPI_NONE)
    torch.cuda.synchronize()
    ref = moe.gmm(a, None, 1, codes, scales, offs, moe.EPI_NONE)
    assert_rows_close(host_f64(out), ref)


def test_combine_identity_and_weighted():
    T, k, H = 37, 3, 64
    logits = synth.router_logits(T, 8, 0, 47)
    rt = _route(logits, k)
    ref_rt = moe.route(logits, k)
    o = synth.bf16_normal((T * k, H), 0, 48)
    y = api.moe_combine(dev_bf16(o), rt.topk_w, rt.pair_pos)
    torch.cuda.synchronize()
    ref = moe.combine(bf16.to_f64(o), ref_rt.topk_w, ref_rt.pair_pos, T, k)
    assert_rows_close(host_f64(y), ref)
    # k = 1 with weight 1: combine after permute is the identity, bit for bit
    rt1 = _route(logits, 1)
    perm = rt1.sorted_pair.cpu().numpy()
    x = synth.bf16_normal((T, H), 0, 49)
    y1 = api.moe_combine(dev_bf16(x[perm]), rt1.topk_w, rt1.pair_pos)
    assert np.array_equal(y1.cpu().view(torch.int16).numpy().view(np.uint16), x)


def _layer(case, tokens=None):
    layer = api.MoELayer(dev_u32(case.gu_codes), dev_bf16(case.gu_scales), dev_u32(case.dn_codes),
                         dev_bf16(case.dn_scales), case.T, case.k)
    y = layer(dev_bf16(case.x), dev_f32(case.logits))
    torch.cuda.synchronize()
    ref = moe.moe_layer(case.x, case.logits, case.gu_codes, case.gu_scales, case.dn_codes,
                        case.dn_scales, case.k, tokens=tokens)
    return layer, y, ref


def test_moe_decode_layer_full_config():
    """64 tokens, 128 experts, top-8, hidden 2816, expert intermediate 704."""
    case = synth.case_moe_decode()
    layer, y, ref = _layer(case)
    assert np.array_equal(layer.rt.sorted_pair.cpu().numpy(), ref.routing.sorted_pair)
    assert_rows_close(host_f64(layer.h), ref.h, what="h")
    assert_rows_close(host_f64(y), ref.y, what="y")


@pytest.mark.parametrize("T", [1, 2, 3])
def test_moe_small_batch_split_k(T):
    """A few decode tokens through the full-size layer.  One token's 8 routed rows give the
    gate/up GEMM only 88 units, so it splits K in three (the workspace then holds the float32
    partials) and the last split of each tile reduces them and applies the GELU gate; 16 and 24
    rows already fill more than half of the pipelines and take the unsplit path."""
    case = synth.moe_case(T, 128, 8, 2816, 704, seed=90 + T)
    rows = T * 8
    # prepared records: one per (8-row token block, 512-k stage) of 8 x 1088 bytes of fp16 rows,
    # 16 x 4 quads of 16 bytes and 8 multipliers; at most min(rows, rows // 8 + 128) blocks
    blocks = min(rows, rows // 8 + min(128, rows))
    prepared = blocks * ((2816 // 32 + 15) // 16) * (8 * 1088 + 16 * 4 * 16 + 8 * 4)
    ws = api.w4_workspace_bytes(_lib.W4_OP_GMM, rows, 2 * 704, 2816, 128, 8)
    if T == 1:
        assert ws > prepared + 3 * 4 * rows * 1408
    else:
        assert ws <= prepared + 256
    layer, y, ref = _layer(case)
    assert_rows_close(host_f64(layer.h), ref.h, what="h")
    assert_rows_close(host_f64(y), ref.y, what="y")


def test_moe_prefill_layer_sampled_tokens():
    """8192 tokens with Zipf(1.1)-skewed experts; 40 tokens checked, including the ones routed to
    the most and least loaded experts."""
    case = synth.case_moe_prefill()
    rt = moe.route(case.logits, case.k)
    hot, cold = int(np.argmax(rt.counts)), int(np.argmin(np.where(rt.counts > 0, rt.counts, 1 << 30)))
    ids = rt.topk_ids
    pick = [int(np.nonzero((ids == hot).any(1))[0][0]), int(np.nonzero((ids == cold).any(1))[0][0])]
    rng = np.random.default_rng(51)
    tokens = np.unique(np.concatenate([pick, [0, case.T - 1], rng.choice(case.T, 36, replace=False)]))
    layer, y, ref = _layer(case, tokens)
    assert np.array_equal(layer.rt.expert_offsets.cpu().numpy(), rt.expert_offsets)
    assert_rows_close(host_f64(y)[tokens], ref.y[tokens])


def test_moe_prefill_layer_every_row():
    """The prefill layer (8192 tokens, 128 Zipf(1.1)-skewed experts: hot experts with thousands
    of rows, cold ones with a few, ragged last blocks) through the tensor-core kernel, checked on
    every routed row: all 65,536 rows of h against the oracle's grouped GEMM with the GELU gate,
    and all 65,536 rows of o against the oracle's down GEMM fed the device's own h (expert by
    expert, so that only one chunk of float64 rows is held at a time)."""
    case = synth.case_moe_prefill()
    ref_rt = moe.route(case.logits, case.k)
    dev = torch.device("cuda")
    layer = api.MoELayer(dev_u32(case.gu_codes), dev_bf16(case.gu_scales), dev_u32(case.dn_codes),
                         dev_bf16(case.dn_scales), case.T, case.k)
    layer(dev_bf16(case.x), dev_f32(case.logits))
    torch.cuda.synchronize()
    assert np.array_equal(layer.rt.expert_offsets.cpu().numpy(), ref_rt.expert_offsets)
    assert np.array_equal(layer.rt.sorted_pair.cpu().numpy(), ref_rt.sorted_pair)
    counts = np.diff(ref_rt.expert_offsets)
    assert counts.max() > 1000 and counts[counts > 0].min() < 10
    h_ref = moe.gmm(case.x, ref_rt.sorted_pair, case.k, case.gu_codes, case.gu_scales,
                    ref_rt.expert_offsets, moe.EPI_GELU_GATE)
    assert_rows_close(host_f64(layer.h), h_ref, what="h")
    del h_ref
    h_bits = layer.h.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    o_dev = host_f64(layer.o)
    off = ref_rt.expert_offsets.astype(np.int64)
    e0 = 0
    while e0 < case.E:
        e1 = e0 + 1
        while e1 < case.E and off[e1 + 1] - off[e0] <= 8192:
            e1 += 1
        r0, r1 = int(off[e0]), int(off[e1])
        if r1 > r0:
            o_ref = moe.gmm(h_bits[r0:r1], None, 1, case.dn_codes[e0:e1], case.dn_scales[e0:e1],
                            off[e0:e1 + 1] - r0, moe.EPI_NONE)
            assert_rows_close(o_dev[r0:r1], o_ref, what=f"o (experts {e0}..{e1 - 1})")
        e0 = e1


@pytest.mark.parametrize("T,H", [(1, 2816), (37, 2816), (256, 2816), (5, 8), (3, 4104)])
def test_rms_chain_matches_oracle(T, H):
    """moe_rms_chain against oracle.moe.rms_chain: every element within one bf16 unit (float32
    sum of squares and quotient on the device, float64 in the oracle) and at least 99.9% of them
    bit-identical."""
    y = synth.bf16_normal((T, H), 0, 900 + T)
    y = bf16.from_f64(bf16.to_f64(y) * (1 + np.arange(T)[:, None]))     # rows of different scale
    x = api.moe_rms_chain(dev_bf16(y))
    torch.cuda.synchronize()
    got = x.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    ref = moe.rms_chain(y)
    assert np.all(np.abs(got.astype(np.int32) - ref.astype(np.int32)) <= 1)
    assert np.mean(got == ref) >= 0.999
