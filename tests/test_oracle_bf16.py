"""Pins for the oracle's bf16 conversions (CPU only).

bf16 is the storage type of activations and scales on "Repacked QAT Gemma 4 26B-A4B serves on
one TPU v6e at 1.9x FP8 throughput", section "A repack, not a re-quantization".  The pins are
the format's own definition: float32 -> bf16 rounding as done by a library (torch), exact
midpoint cases, overflow, and the exhaustive round trip over all 65536 patterns.
"""
import numpy as np
import torch

from oracle import bf16


def _torch_bf16_bits(x32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_matches_library_rounding_of_float32_values():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 1 << 32, size=200_000, dtype=np.uint64).astype(np.uint32)
    x32 = bits.view(np.float32)
    x32 = x32[np.isfinite(x32)]
    # values near the top of the range: torch saturates differently only for NaN; keep finite
    got = bf16.from_f64(x32.astype(np.float64))
    want = _torch_bf16_bits(x32)
    assert np.array_equal(got, want)


def test_exact_midpoints_round_to_even_and_no_double_rounding():
    one = 1.0
    # 1 + 2^-8 is halfway between 1 (0x3F80, even) and 1 + 2^-7 (0x3F81): ties to even
    assert bf16.from_f64(np.array([one + 2.0 ** -8]))[0] == 0x3F80
    # 1 + 3*2^-8 is halfway between 0x3F81 (odd) and 0x3F82 (even)
    assert bf16.from_f64(np.array([one + 3 * 2.0 ** -8]))[0] == 0x3F82
    # just above the midpoint rounds up; a detour through float32 would lose 2^-40 and tie
    assert bf16.from_f64(np.array([one + 2.0 ** -8 + 2.0 ** -40]))[0] == 0x3F81
    assert bf16.from_f64(np.array([-(one + 2.0 ** -8 + 2.0 ** -40)]))[0] == 0xBF81


def test_known_patterns_and_specials():
    assert bf16.to_f64(np.array([0x3F80]))[0] == 1.0
    assert bf16.to_f64(np.array([0xC100]))[0] == -8.0
    assert bf16.to_f64(np.array([0x0001]))[0] == 2.0 ** -133      # smallest subnormal
    assert np.isinf(bf16.to_f64(np.array([0x7F80]))[0])
    assert bf16.from_f64(np.array([np.nan]))[0] == 0x7FC0
    assert bf16.from_f64(np.array([np.inf]))[0] == 0x7F80
    assert bf16.from_f64(np.array([-0.0]))[0] == 0x8000
    assert bf16.from_f64(np.array([2.0 ** -134]))[0] == 0x0000      # half the smallest: tie to 0
    assert bf16.from_f64(np.array([1.5 * 2.0 ** -133]))[0] == 0x0002  # tie to even (2)
    top = (2.0 - 2.0 ** -7) * 2.0 ** 127
    half_ulp = 2.0 ** (127 - 8)
    assert bf16.from_f64(np.array([top]))[0] == 0x7F7F
    assert bf16.from_f64(np.array([top + half_ulp * 0.999]))[0] == 0x7F7F
    assert bf16.from_f64(np.array([top + half_ulp]))[0] == 0x7F80     # tie rounds to even -> inf


def test_exhaustive_round_trip():
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    x = bf16.to_f64(b)
    keep = ~np.isnan(x)
    assert np.array_equal(bf16.from_f64(x[keep]), b[keep])
