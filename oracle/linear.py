"""Weight-only W4A16 dense linear.  Test infrastructure only.

Source: "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", section
"What changed in vLLM's TPU backend" (W4A16 for linear layers; per-32 scales; weights
dequantised before the multiply; activations stay bf16, so quantisation is weight-only), and
"What quantization really is", section "What you choose to shrink" (W4A16: 4-bit weights,
16-bit activations).

y[m, n] = sum_k x[m, k] * s[n, k // 32] * q[n, k], evaluated in float64 and left unrounded.
"""
from __future__ import annotations

import numpy as np

from . import bf16, q4


def w4a16_linear(x_bits, codes, scales) -> np.ndarray:
    """x [M, K] bf16 patterns, codes [N, K/8] uint32, scales [N, K/32] bf16 -> y [M, N] float64."""
    x = bf16.to_f64(np.asarray(x_bits, dtype=np.uint16))
    W = q4.dequant(codes, scales)                 # [N, K]
    assert x.shape[1] == W.shape[1]
    return x @ W.T


def w4a16_linear_rows(x_bits, codes, scales, rows) -> np.ndarray:
    """Selected output columns n in ``rows`` only: y[:, rows] (for sampled checks at full size)."""
    rows = np.asarray(rows, dtype=np.int64)
    x = bf16.to_f64(np.asarray(x_bits, dtype=np.uint16))
    W = q4.dequant(np.asarray(codes)[rows], np.asarray(scales)[rows])
    return x @ W.T
