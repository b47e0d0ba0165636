"""Pins for the oracle's weight-format variants (other group sizes, asymmetric zero-point).

Source: "What quantization really is", section "How the ruler works" (asymmetric quantisation
adds a zero-point; group-wise granularity).  Pins:
  * z = 8 and G = 32 is exactly the symmetric Q4_0 oracle (oracle.q4.dequant); z = 8 at a
    larger G is the symmetric oracle with each scale repeated over G / 32 groups;
  * a hand-worked asymmetric group (tests/golden/asym_group.txt);
  * weights planted exactly on an asymmetric grid whose codes span 0..15 round-trip bit for bit;
  * the linear against loops over hand-decoded nibbles with per-group zero-points.
"""
import os

import numpy as np

from oracle import bf16, q4, variants
from w4a16_group_quantized_w4_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_symmetric_special_case_is_the_q4_oracle():
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 1 << 32, size=(6, 16), dtype=np.uint64).astype(np.uint32)   # K = 128
    s32 = synth.abs_normal_scales((6, 4), 0.02, 1e-3, 0, 4)
    assert np.array_equal(variants.dequant(codes, s32, 32), q4.dequant(codes, s32))
    z8 = np.full((6, 4), 8, np.uint8)
    assert np.array_equal(variants.dequant(codes, s32, 32, z8), q4.dequant(codes, s32))
    s64 = synth.abs_normal_scales((6, 2), 0.02, 1e-3, 0, 5)
    assert np.array_equal(variants.dequant(codes, s64, 64), q4.dequant(codes, np.repeat(s64, 2, axis=1)))
    s128 = s64[:, :1]
    assert np.array_equal(variants.dequant(codes, s128, 128, np.full((6, 1), 8, np.uint8)),
                          q4.dequant(codes, np.repeat(s128, 4, axis=1)))


def test_hand_worked_asymmetric_group():
    """The golden file lists w (bf16 hex) of one 32-group and the scale, zero-point and codes
    worked by hand from the stated formulas."""
    block = {}
    for line in open(os.path.join(GOLDEN, "asym_group.txt")):
        line = line.split("#")[0].strip()
        if line:
            key, val = line.split(":")
            block[key.strip()] = val.split()
    w = np.array([int(v, 16) for v in block["w"]], dtype=np.uint16)[None, :]
    qz = variants.quantize_asym(w, 32)
    assert int(qz.scales[0, 0]) == int(block["scale"][0], 16)
    assert int(qz.zeros[0, 0]) == int(block["zero"][0])
    assert list(qz.u[0]) == [int(v) for v in block["u"]]


def test_planted_asymmetric_grid_round_trips():
    rng = np.random.default_rng(8)
    R, K, G = 5, 256, 64
    ng = K // G
    u = rng.integers(0, 16, size=(R, ng, G))
    u[:, :, 0], u[:, :, 1] = 0, 15                      # every group spans the whole 0..15 range
    z = rng.integers(0, 16, size=(R, ng))
    # scales 15 * s exactly representable and (hi - lo) / 15 = s exactly: s = m * 2^e, m < 2^4
    s_bits = bf16.from_f64(rng.integers(1, 16, size=(R, ng)) * 2.0 ** rng.integers(-12, -4, size=(R, ng)))
    s = bf16.to_f64(s_bits)
    w = (u - z[:, :, None]) * s[:, :, None]
    w_bits = bf16.from_f64(w.reshape(R, K))
    assert np.array_equal(bf16.to_f64(w_bits), w.reshape(R, K))     # the planted values are bf16
    qz = variants.quantize_asym(w_bits, G)
    assert np.array_equal(qz.scales, s_bits)
    assert np.array_equal(qz.zeros, z.astype(np.uint8))
    assert np.array_equal(qz.u, u.reshape(R, K))
    assert np.array_equal(variants.dequant(qz.codes, qz.scales, G, qz.zeros), w.reshape(R, K))


def test_linear_against_loops_with_hand_decoded_nibbles():
    rng = np.random.default_rng(21)
    M, N, K, G = 3, 5, 128, 64
    x_bits = synth.bf16_normal((M, K), 0, 22)
    words = rng.integers(0, 1 << 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    s_bits = bf16.from_f64(rng.uniform(0.01, 0.1, size=(N, K // G)))
    zeros = rng.integers(0, 16, size=(N, K // G)).astype(np.uint8)
    y = variants.linear(x_bits, words, s_bits, G, zeros)
    xf = bf16.to_f64(x_bits)
    sf = bf16.to_f64(s_bits)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                u = (int(words[n, k // 8]) >> (4 * (k % 8))) & 0xF
                acc += xf[m, k] * sf[n, k // G] * (u - int(zeros[n, k // G]))
            assert abs(acc - y[m, n]) <= 1e-12 * (1 + abs(acc))
