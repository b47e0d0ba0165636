"""Variants of the weight format: other group sizes along K and an asymmetric zero-point.
Test infrastructure only.

Source: "What quantization really is", section "How the ruler works": quantisation stores a
scale and an optional zero-point; when values are not centred on zero, asymmetric quantisation
adds a zero-point; a shared scale and zero-point can cover a whole tensor, a channel, a token or a
small group (group-wise granularity), the standard uniform formulas used across LLM papers.  The
page's formulas are lost in extraction; the readings taken are the standard uniform ones:

  * codes are unsigned 4-bit u in 0..15, packed as in layout L1 (nibble j of a word = element j);
  * one bf16 scale s and, for the asymmetric form, one integer zero-point z in 0..15 per group of
    G consecutive elements along the input dimension (G a multiple of 32);
  * dequantised weight W = s * (u - z); the symmetric Q4_0 grid of the main path is the special
    case z = 8 (q = u - 8 in -8..7) with G = 32;
  * asymmetric quantisation of a group (used to make test data): lo = min w, hi = max w,
    s = bf16((hi - lo) / 15), z = clamp(rint(-lo / s), 0, 15), u = clamp(rint(w / s) + z, 0, 15),
    float64 arithmetic on the bf16 values, rint = round half to even; a group with hi == lo
    (s = 0) gets u = z = 0.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import bf16, q4

NIBBLES = 16


def unsigned_codes(codes) -> np.ndarray:
    """Packed words [R, K/8] -> unsigned codes u [R, K] in 0..15 (layout L1)."""
    return q4.unpack(codes) + 8


def pack_unsigned(u) -> np.ndarray:
    """Unsigned codes u [R, K] in 0..15 -> packed words [R, K/8] (layout L1)."""
    u = np.asarray(u, dtype=np.int64)
    assert u.min(initial=0) >= 0 and u.max(initial=0) < NIBBLES
    return q4.pack(u - 8)


def dequant(codes, scales, group: int, zeros=None) -> np.ndarray:
    """W[n, k] = s[n, k // G] * (u[n, k] - z[n, k // G]) in float64 (exact).

    codes [..., N, K/8] uint32, scales [..., N, K/G] bf16 patterns, zeros [..., N, K/G] uint8 or
    None (z = 8, the symmetric grid)."""
    codes = np.asarray(codes)
    scales = np.asarray(scales)
    lead = codes.shape[:-1]
    u = unsigned_codes(codes.reshape(-1, codes.shape[-1]))
    K = u.shape[1]
    assert group % q4.GROUP == 0 and K % group == 0
    s = bf16.to_f64(scales.reshape(-1, scales.shape[-1]))
    assert s.shape[1] * group == K
    if zeros is None:
        z = np.full(s.shape, 8.0)
    else:
        z = np.asarray(zeros).reshape(-1, s.shape[1]).astype(np.float64)
    W = (u.astype(np.float64) - np.repeat(z, group, axis=1)) * np.repeat(s, group, axis=1)
    return W.reshape(*lead, K)


@dataclass
class Quantized:
    codes: np.ndarray      # uint32 [R, K/8]
    scales: np.ndarray     # uint16 [R, K/G] bf16 patterns
    zeros: np.ndarray      # uint8  [R, K/G]
    u: np.ndarray          # int64  [R, K]


def quantize_asym(w_bits, group: int) -> Quantized:
    """Asymmetric 4-bit quantisation of bf16 weights [R, K] with one scale and zero-point per
    group of G along K (the reading stated in the module docstring)."""
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    R, K = w_bits.shape
    assert K % group == 0
    w = bf16.to_f64(w_bits).reshape(-1, group)
    lo, hi = w.min(axis=1), w.max(axis=1)
    s_bits = bf16.from_f64((hi - lo) / 15.0)
    s = bf16.to_f64(s_bits)
    nz = s > 0
    z = np.zeros(w.shape[0])
    u = np.zeros(w.shape, dtype=np.int64)
    z[nz] = np.clip(np.rint(-lo[nz] / s[nz]), 0, 15)
    u[nz] = np.clip(np.rint(w[nz] / s[nz, None]) + z[nz, None], 0, 15).astype(np.int64)
    u = u.reshape(R, K)
    return Quantized(codes=pack_unsigned(u), scales=s_bits.reshape(R, K // group),
                     zeros=z.astype(np.uint8).reshape(R, K // group), u=u)


def linear(x_bits, codes, scales, group: int, zeros=None) -> np.ndarray:
    """y [M, N] = x [M, K] @ W^T in float64 with W = dequant(codes, scales, group, zeros)."""
    x = bf16.to_f64(np.asarray(x_bits, dtype=np.uint16))
    W = dequant(codes, scales, group, zeros)
    assert x.shape[1] == W.shape[1]
    return x @ W.T


def gmm(a_bits, a_row_of_pair, k: int, codes, scales, expert_offsets, epilogue: int, group: int,
        zeros=None) -> np.ndarray:
    """The grouped GEMM of oracle.moe.gmm on the variant format: expert e's weights are
    dequant(codes[e], scales[e], group, zeros[e]); gate/up split and GELU gate as there."""
    from . import moe
    a = bf16.to_f64(np.asarray(a_bits, dtype=np.uint16))
    codes = np.asarray(codes)
    off = np.asarray(expert_offsets, dtype=np.int64)
    E, N = codes.shape[0], codes.shape[1]
    N_out = N // 2 if epilogue == moe.EPI_GELU_GATE else N
    out = np.full((int(off[-1]), N_out), np.nan)
    for e in range(E):
        r = np.arange(off[e], off[e + 1])
        if r.size == 0:
            continue
        src = (np.asarray(a_row_of_pair)[r] // k) if a_row_of_pair is not None else r
        W = dequant(codes[e], np.asarray(scales)[e], group, None if zeros is None else np.asarray(zeros)[e])
        Y = a[src] @ W.T
        if epilogue == moe.EPI_GELU_GATE:
            I = N // 2
            Y = moe.gelu_tanh(Y[:, :I]) * Y[:, I:]
        out[r] = Y
    return out
