"""Pins for the oracle's W4A16 dense linear (CPU only).

Definition ("Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", section
"What changed in vLLM's TPU backend": per-32 scales, weights dequantised before the multiply,
bf16 activations): y[m, n] = sum_k x[m, k] * s[n, k // 32] * q[n, k].

Pins: exact integer arithmetic (x small integers, s powers of two), a constant-weight closed
form, one-hot probes that read single weights back, and a loop-by-loop brute force with the
nibble layout decoded by hand on non-square shapes (a transposed operand or a wrong group
offset fails these).
"""
from fractions import Fraction

import numpy as np

from oracle import bf16, linear, q4
from w4a16_group_quantized_w4_b200 import synth


def _bf16(x):
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def test_exact_integer_case():
    rng = np.random.default_rng(11)
    M, N, K = 3, 5, 96
    x = rng.integers(-4, 5, size=(M, K))
    q = rng.integers(-8, 8, size=(N, K))
    e = rng.integers(0, 6, size=(N, K // 32))
    s = 2.0 ** (-e)
    y = linear.w4a16_linear(_bf16(x), q4.pack(q), _bf16(s))
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(int(x[m, k])) * Fraction(1, 2 ** int(e[n, k // 32])) * int(q[n, k])
                        for k in range(K))
            assert Fraction(y[m, n]) == exact


def test_constant_weight_closed_form():
    rng = np.random.default_rng(12)
    x_bits = synth.bf16_normal((4, 128), 0, 12)
    c, s = -3, 0.015625
    q = np.full((6, 128), c)
    y = linear.w4a16_linear(x_bits, q4.pack(q), _bf16(np.full((6, 4), s)))
    xs = bf16.to_f64(x_bits).sum(axis=1)
    assert np.allclose(y, (s * c * xs)[:, None], rtol=1e-12, atol=1e-12)


def test_one_hot_probe_reads_each_weight():
    rng = np.random.default_rng(13)
    N, K = 4, 64
    q = rng.integers(-8, 8, size=(N, K))
    s = rng.uniform(0.1, 2.0, size=(N, K // 32))
    s_bits = _bf16(s)
    s_val = bf16.to_f64(s_bits)
    x = np.eye(K)
    y = linear.w4a16_linear(_bf16(x), q4.pack(q), s_bits)   # y[k, n] = s[n, k//32] q[n, k]
    for k in range(K):
        for n in range(N):
            assert y[k, n] == s_val[n, k // 32] * q[n, k]


def test_brute_force_loops_with_hand_decoded_nibbles():
    rng = np.random.default_rng(14)
    M, N, K = 5, 7, 64
    x_bits = synth.bf16_normal((M, K), 0, 14)
    words = rng.integers(0, 1 << 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    s_bits = _bf16(rng.uniform(0.01, 0.1, size=(N, K // 32)))
    y = linear.w4a16_linear(x_bits, words, s_bits)
    xf = [[float(v) for v in row] for row in bf16.to_f64(x_bits)]
    sf = bf16.to_f64(s_bits)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                word = int(words[n, k // 8])
                j = k % 8
                u = (word >> (4 * j)) & 0xF                        # layout L1: nibble j = element j
                acc += xf[m][k] * float(sf[n, k // 32]) * (u - 8)
            assert abs(acc - y[m, n]) <= 1e-12 * (1 + abs(acc))


def test_selected_rows_match_full():
    case = synth.dense_case(2, 48, 128, 0.02, 1e-3, seed=3)
    full = linear.w4a16_linear(case.x, case.codes, case.scales)
    rows = np.array([0, 5, 47])
    part = linear.w4a16_linear_rows(case.x, case.codes, case.scales, rows)
    assert np.array_equal(part, full[:, rows])
