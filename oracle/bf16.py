"""bf16 <-> float64 for the oracle.  Test infrastructure only.

bf16 is the storage type the pages give for activations and for the per-group scales ("storing
the scale at bf16, the precision vLLM's TPU W4A16 layers load it at": "Repacked QAT Gemma 4
26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", section "A repack, not a
re-quantization").  A bf16 value is an IEEE binary32 with the low 16 bits of the significand
dropped: 1 sign bit, 8 exponent bits, 7 stored significand bits.
"""
from __future__ import annotations

import numpy as np

BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127
QNAN_BITS = 0x7FC0


def to_f64(bits) -> np.ndarray:
    """bf16 patterns (uint16) -> float64, exactly: the pattern is the top half of a binary32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):                # signalling-NaN patterns widen to NaN
        return b.view(np.float32).astype(np.float64)


def from_f64(x) -> np.ndarray:
    """float64 -> bf16 pattern, rounding once to the nearest bf16 value, ties to even.

    Written from the definition, without passing through float32 (two roundings would differ
    at bf16 midpoints).  A finite value is a significand k times a power of two 2^e; a bf16
    significand has 8 bits for normal numbers and the quantum never goes below 2^-133
    (subnormals).  Results past the largest finite bf16 become infinity, NaN becomes the quiet
    NaN 0x7FC0.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    nan = np.isnan(x)
    ax = np.abs(np.where(nan, 0.0, x))
    with np.errstate(over="ignore", invalid="ignore"):
        _, e = np.frexp(ax)                      # ax = f * 2^e, f in [0.5, 1)
        qe = np.maximum(e - 8, -133)             # quantum of the bf16 binade holding ax
        k = np.rint(np.ldexp(ax, -qe))           # exact scaling, then nearest-even integer
        val = np.ldexp(k, qe)                    # the rounded magnitude (exact in float64)
        val = np.where(np.isinf(ax) | (val > BF16_MAX), np.inf, val)
        bits = (val.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    sign = np.signbit(x) & ~nan
    bits = np.where(sign, bits | np.uint16(0x8000), bits)
    out[...] = np.where(nan, np.uint16(QNAN_BITS), bits)
    return out
