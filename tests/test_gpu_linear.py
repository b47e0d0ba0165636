"""GPU parity of w4a16_linear against the float64 oracle.

Definition: "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", section
"What changed in vLLM's TPU backend" (W4A16 linear: per-32 scales, weights dequantised on chip,
bf16 activations).  Tolerance per output row: rel-L2 <= 5e-3 and max-abs <= 2e-2 * max|y_ref|;
the exact-integer case is compared bit for bit.
"""
import numpy as np
import pytest
import torch

from oracle import bf16, linear, q4
from w4a16_group_quantized_w4_b200 import api, synth
from tests._util import assert_rows_close, dev_bf16, dev_u32, host_bf16_bits, host_f64

pytestmark = pytest.mark.gpu


def _run(case):
    y = api.w4a16_linear(dev_bf16(case.x), dev_u32(case.codes), dev_bf16(case.scales))
    torch.cuda.synchronize()
    return y


def test_dense_small_config():
    case = synth.case_dense_small()
    ref = linear.w4a16_linear(case.x, case.codes, case.scales)
    assert_rows_close(host_f64(_run(case)), ref)


@pytest.mark.parametrize("M,N,K", [(1, 8, 32), (3, 13, 96), (5, 200, 256), (16, 64, 2816),
                                   (33, 136, 704), (64, 256, 512), (100, 128, 4096), (1, 1, 64)])
def test_ragged_shapes(M, N, K):
    case = synth.dense_case(M, N, K, 0.02, 1e-3, seed=M * 7 + N)
    ref = linear.w4a16_linear(case.x, case.codes, case.scales)
    assert_rows_close(host_f64(_run(case)), ref)


def test_exact_integer_case_bit_exact():
    """x with at most 16 nonzero entries of +-1 per row and power-of-two scales: y is an integer
    multiple of a power of two below 2^8 in magnitude, so bf16 holds it exactly."""
    rng = np.random.default_rng(31)
    M, N, K = 8, 384, 1024
    x = np.zeros((M, K), np.float32)
    for m in range(M):
        idx = rng.choice(K, size=16, replace=False)
        x[m, idx] = rng.choice([-1.0, 1.0], size=16)
    q = rng.integers(-8, 8, size=(N, K))
    s = np.full((N, K // 32), 0.125, np.float32)
    x_bits = synth.f32_to_bf16_bits(x)
    codes = q4.pack(q)
    s_bits = synth.f32_to_bf16_bits(s)
    ref = linear.w4a16_linear(x_bits, codes, s_bits)
    y = api.w4a16_linear(dev_bf16(x_bits), dev_u32(codes), dev_bf16(s_bits))
    assert np.array_equal(host_bf16_bits(y), bf16.from_f64(ref))


def test_zero_rows():
    case = synth.dense_case(0, 64, 256, 0.02, 1e-3, seed=1)
    y = api.w4a16_linear(dev_bf16(case.x), dev_u32(case.codes), dev_bf16(case.scales))
    assert y.shape == (0, 64)


@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_gemv_full_size_sampled(M):
    """K=4096, N=14336 at full size; 160 sampled output columns checked against the oracle."""
    case = synth.case_dense_gemv(M)
    y = host_f64(_run(case))
    rng = np.random.default_rng(M)
    cols = np.unique(np.concatenate([[0, 127, 128, 14335], rng.choice(14336, 156, replace=False)]))
    ref = linear.w4a16_linear_rows(case.x, case.codes, case.scales, cols)
    assert_rows_close(y[:, cols], ref)


def test_repeat_calls_are_deterministic():
    case = synth.case_dense_gemv(4)
    y1 = host_bf16_bits(_run(case))
    y2 = host_bf16_bits(_run(case))
    assert np.array_equal(y1, y2)


def test_workspace_reused_across_shapes_with_stale_contents():
    """One workspace filled with garbage and shared by split-K calls of different shapes."""
    from w4a16_group_quantized_w4_b200 import _lib
    shapes = [(1, 14336, 4096), (4, 14336, 4096), (16, 14336, 4096), (3, 2048, 2816), (1, 14336, 4096)]
    need = max(api.w4_workspace_bytes(_lib.W4_OP_LINEAR, M, N, K, 1, 1) for M, N, K in shapes)
    assert need > 0
    ws = torch.full((need,), 0xA5, dtype=torch.uint8, device="cuda")
    for i, (M, N, K) in enumerate(shapes):
        case = synth.dense_case(M, N, K, 0.01, 1e-4, seed=40 + i)
        y = api.w4a16_linear(dev_bf16(case.x), dev_u32(case.codes), dev_bf16(case.scales), ws=ws)
        torch.cuda.synchronize()
        cols = np.arange(0, N, 97)
        ref = linear.w4a16_linear_rows(case.x, case.codes, case.scales, cols)
        assert_rows_close(host_f64(y)[:, cols], ref)


def _golden_words():
    """(codes q_0..q_7, word) pairs worked by hand in tests/golden/nibble_layout.txt (layout L1)."""
    import os
    out = []
    for line in open(os.path.join(os.path.dirname(__file__), "golden", "nibble_layout.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        lhs, rhs = line.split("->")
        out.append(([int(v) for v in lhs.split()], int(rhs, 16)))
    return out


@pytest.mark.parametrize("M", [16, 64])          # weight-streaming kernel, tensor-core kernel
def test_golden_l1_words_through_linear(M):
    """Hand-packed layout-L1 words (not produced by the oracle) as the weights of a linear with
    scale 1 and one-hot activation rows: y[m, n] must be exactly code m of row n, as the golden
    file lists it.  A kernel that read the nibbles in any other order fails this bit for bit."""
    gold = _golden_words()
    N, K = 128, 64
    words = np.empty((N, K // 8), np.uint32)
    q = np.empty((N, K), np.int64)
    for n in range(N):
        for w in range(K // 8):
            codes, word = gold[(n * 3 + w) % len(gold)]
            words[n, w] = word
            q[n, 8 * w:8 * w + 8] = codes
    x = np.eye(K, dtype=np.float32)[np.arange(M) % K]
    s_bits = synth.f32_to_bf16_bits(np.ones((N, K // 32), np.float32))
    y = api.w4a16_linear(dev_bf16(synth.f32_to_bf16_bits(x)), dev_u32(words), dev_bf16(s_bits))
    torch.cuda.synchronize()
    expect = q[:, np.arange(M) % K].T.astype(np.float64)
    assert np.array_equal(host_f64(y), expect)


def test_workspace_cache_per_stream_and_kept_alive():
    """Scratch is shared only by calls on one stream, and an outgrown buffer stays allocated (a
    CUDA graph captured with it keeps a valid pointer)."""
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    a = api.workspace(1000, "cuda", s1)
    b = api.workspace(1000, "cuda", s2)
    assert a.data_ptr() != b.data_ptr()
    assert api.workspace(500, "cuda", s1) is a
    ptr_a = a.data_ptr()
    c = api.workspace(a.numel() + (1 << 20), "cuda", s1)      # outgrows s1's buffer
    assert c.data_ptr() != ptr_a and c.numel() >= a.numel() + (1 << 20)
    assert api.workspace(500, "cuda", s1) is c
    key = (torch.device("cuda", torch.cuda.current_device()), s1.cuda_stream)
    assert any(t.data_ptr() == ptr_a for t in api._WS[key])
