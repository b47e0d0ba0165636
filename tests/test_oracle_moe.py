"""Pins for the oracle's routing, grouped GEMM, GELU gate and combine (CPU only).

The pages give "128 experts per layer and 8 active per token" ("Repacked QAT Gemma 4 26B-A4B
serves on one TPU v6e at 1.9x FP8 throughput", section "The gap at 26B") and a grouped matmul
over the experts' packed int4 weights with per-32 scales (section "What changed in vLLM's TPU
backend").  The router math, the gate/up split and the activation are not on the pages; they
are pinned here to library routines (softmax, sorting, erf, PyTorch's tanh-approximate GELU)
and to mathematical identities.  No page value exists for the tanh-GELU gate; it is pinned to
an independent implementation of the same published approximation.
"""
import math

import numpy as np
import pytest
import torch

from oracle import bf16, linear, moe, q4
from w4a16_group_quantized_w4_b200 import synth


def _bf16(x):
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def test_k1_is_argmax_with_unit_weight():
    lg = synth.router_logits(200, 128, 0, 1)
    rt = moe.route(lg, 1)
    assert np.array_equal(rt.topk_ids[:, 0], np.argmax(lg, axis=1))
    assert (rt.topk_w == 1.0).all()


def test_k_equals_E_gives_full_softmax():
    lg = synth.router_logits(50, 16, 0, 2)
    rt = moe.route(lg, 16)
    sm = torch.softmax(torch.from_numpy(lg.astype(np.float64)), dim=1).numpy()
    assert np.allclose(np.take_along_axis(sm, rt.topk_ids.astype(np.int64), 1), rt.topk_w,
                       rtol=1e-13, atol=0)


def test_weights_are_renormalised_full_softmax():
    lg = synth.router_logits(300, 128, 0, 3)
    rt = moe.route(lg, 8)
    sm = torch.softmax(torch.from_numpy(lg.astype(np.float64)), dim=1).numpy()
    sel = np.take_along_axis(sm, rt.topk_ids.astype(np.int64), 1)
    assert np.allclose(sel / sel.sum(1, keepdims=True), rt.topk_w, rtol=1e-12, atol=0)
    assert (np.diff(rt.topk_w, axis=1) <= 0).all()


def test_selection_matches_sorted_brute_force_and_ties_go_low():
    rng = np.random.default_rng(21)
    lg = rng.integers(-3, 4, size=(64, 16)).astype(np.float32)   # many equal logits
    rt = moe.route(lg, 5)
    for t in range(64):
        order = sorted(range(16), key=lambda e: (-float(lg[t, e]), e))
        assert rt.topk_ids[t].tolist() == order[:5]


def test_permutation_is_stable_counting_sort():
    lg = synth.router_logits(97, 32, 0, 4)
    k = 4
    rt = moe.route(lg, k)
    flat = rt.topk_ids.reshape(-1)
    want = sorted(range(97 * k), key=lambda p: (int(flat[p]), p))
    assert rt.sorted_pair.tolist() == want
    assert np.array_equal(rt.pair_pos[rt.sorted_pair], np.arange(97 * k))
    counts = np.array([(flat == e).sum() for e in range(32)])
    assert np.array_equal(np.diff(rt.expert_offsets), counts)
    assert rt.expert_offsets[0] == 0 and rt.expert_offsets[-1] == 97 * k


def test_gelu_identities_and_erf_form():
    z = np.linspace(-12, 12, 4001)
    g = moe.gelu_tanh(z)
    # z/2 (1 + tanh(c(z + a z^3))) - (-z)/2 (1 + tanh(-c(z + a z^3))) = z
    assert np.allclose(g - moe.gelu_tanh(-z), z, rtol=0, atol=1e-12)
    assert moe.gelu_tanh(np.array([0.0]))[0] == 0.0
    erf_form = np.array([0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in z])
    assert np.max(np.abs(g - erf_form)) < 1e-3
    assert abs(g[-1] - 12) < 1e-9 and abs(g[0]) < 1e-9


def test_gelu_matches_an_independent_tanh_gelu():
    """PyTorch's tanh-approximate GELU, a separate implementation of the same published
    approximation (Hendrycks and Gimpel's tanh form), agrees in float64; a wrong cubic
    coefficient or scale would differ by far more than rounding."""
    import torch
    z = np.linspace(-12, 12, 20001)
    ref = torch.nn.functional.gelu(torch.tensor(z, dtype=torch.float64), approximate="tanh").numpy()
    assert np.max(np.abs(moe.gelu_tanh(z) - ref)) < 1e-13


def test_gmm_rows_equal_dense_linear_per_expert():
    rng = np.random.default_rng(22)
    E, N, K, T, k = 3, 16, 64, 10, 2
    a = synth.bf16_normal((T, K), 0, 22)
    codes = rng.integers(0, 1 << 32, size=(E, N, K // 8), dtype=np.uint64).astype(np.uint32)
    scales = _bf16(rng.uniform(0.01, 0.1, size=(E, N, K // 32)))
    lg = synth.router_logits(T, E, 0, 23)
    rt = moe.route(lg, k)
    out = moe.gmm(a, rt.sorted_pair, k, codes, scales, rt.expert_offsets, moe.EPI_NONE)
    for r in range(T * k):
        p = int(rt.sorted_pair[r])
        t, e = p // k, int(rt.topk_ids.reshape(-1)[p])
        y = linear.w4a16_linear(a[t:t + 1], codes[e], scales[e])[0]
        assert np.allclose(out[r], y, rtol=1e-12, atol=1e-15)


def test_gelu_gate_splits_rows_in_halves():
    rng = np.random.default_rng(24)
    E, N, K = 1, 8, 32
    a = synth.bf16_normal((3, K), 0, 24)
    q = rng.integers(-8, 8, size=(N, K))
    s = _bf16(np.full((N, 1), 0.125))
    offs = np.array([0, 3], dtype=np.int32)
    h = moe.gmm(a, None, 1, q4.pack(q)[None], s[None], offs, moe.EPI_GELU_GATE)
    x = bf16.to_f64(a)
    g = x @ (0.125 * q[:4]).T
    u = x @ (0.125 * q[4:]).T
    assert np.allclose(h, moe.gelu_tanh(g) * u, rtol=1e-12, atol=1e-14)


def test_combine_identity_for_one_slot():
    o = synth.bf16_normal((37, 24), 0, 25)
    lg = synth.router_logits(37, 8, 0, 26)
    rt = moe.route(lg, 1)
    o_sorted = o[rt.sorted_pair]                     # permute token rows into expert order
    y = moe.combine(bf16.to_f64(o_sorted), rt.topk_w, rt.pair_pos, 37, 1)
    assert np.array_equal(y, bf16.to_f64(o))


def test_layer_against_per_token_loops():
    rng = np.random.default_rng(27)
    T, E, k, H, I = 6, 5, 2, 64, 32
    case = synth.moe_case(T, E, k, H, I, seed=5)
    res = moe.moe_layer(case.x, case.logits, case.gu_codes, case.gu_scales, case.dn_codes,
                        case.dn_scales, k)
    x = bf16.to_f64(case.x)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(case.logits[t, e]), e))[:k]
        ls = [float(case.logits[t, e]) for e in order]
        ex = [math.exp(v - ls[0]) for v in ls]
        ws = [v / sum(ex) for v in ex]
        y = np.zeros(H)
        for e, wgt in zip(order, ws):
            Wg = q4.dequant(case.gu_codes[e], case.gu_scales[e])
            Wd = q4.dequant(case.dn_codes[e], case.dn_scales[e])
            gu = Wg @ x[t]
            hh = moe.gelu_tanh(gu[:I]) * gu[I:]
            y += wgt * (Wd @ hh)
        assert np.allclose(res.y[t], y, rtol=1e-10, atol=1e-12)
    sub = moe.moe_layer(case.x, case.logits, case.gu_codes, case.gu_scales, case.dn_codes,
                        case.dn_scales, k, tokens=[1, 4])
    assert np.allclose(sub.y[[1, 4]], res.y[[1, 4]], rtol=1e-12, atol=1e-15)
    assert np.isnan(sub.y[0]).all()


def test_zipf_bias_skews_expert_loads():
    lg = synth.router_logits(8192, 128, 0, 102, zipf_s=synth.ZIPF_S)
    rt = moe.route(lg, 8)
    assert rt.counts.max() > 1000 and rt.counts.min() < 10


def test_rms_chain_worked_example():
    """y = [3, 4]: mean(y^2) = 12.5, sqrt(12.5 + 1e-6) = 3.5355340..., so y / rms =
    [0.8485281..., 1.1313708...].  In bf16 (8 significant bits): 0.8485 = 1.69706 * 2^-1 and
    1.69706 * 128 = 217.22 -> 217 / 128 * 2^-1 = 0.84765625 (0x3F59); 1.13137 * 128 = 144.82 ->
    145 / 128 = 1.1328125 (0x3F91)."""
    y = bf16.from_f64(np.array([[3.0, 4.0]]))
    assert list(moe.rms_chain(y)[0]) == [0x3F59, 0x3F91]


def test_rms_chain_constant_rows_and_scale_invariance():
    # a constant row c (|c| >> eps) becomes +-1 exactly
    y = bf16.from_f64(np.array([[2.5] * 64, [-0.375] * 64]))
    x = bf16.to_f64(moe.rms_chain(y))
    assert np.all(x[0] == 1.0) and np.all(x[1] == -1.0)
    # scaling a row by a power of two (exact in bf16) changes nothing while eps stays negligible
    rng = np.random.default_rng(5)
    y = bf16.from_f64(rng.normal(size=(8, 2816)))
    y4 = bf16.from_f64(bf16.to_f64(y) * 4.0)
    assert np.array_equal(moe.rms_chain(y), moe.rms_chain(y4))
    # the output row has mean square 1 up to the bf16 rounding of each element
    x = bf16.to_f64(moe.rms_chain(y))
    assert np.all(np.abs(np.mean(x * x, axis=1) - 1.0) < 2 ** -8)
