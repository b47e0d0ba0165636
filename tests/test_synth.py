"""Checks of the seeded input generators (CPU only): ranges, determinism, counter access."""
import numpy as np

from w4a16_group_quantized_w4_b200 import synth


def test_planted_groups_ranges_and_determinism():
    idx = np.arange(50_000)
    pg = synth.planted_groups(idx, seed=0)
    assert pg.w.shape == (50_000, 32)
    assert synth.log_uniform_check(pg.s) == 1.0
    assert set(np.unique(pg.peak)) == set(range(1, 9))
    assert (np.gcd.reduce(np.abs(pg.q.astype(np.int64)), axis=1) == 1).all()
    assert (pg.q >= -8).all() and (pg.q <= 7).all()
    # the peak level is the largest magnitude and -8 appears exactly when the peak is 8
    assert np.array_equal(np.abs(pg.q.astype(np.int64)).max(axis=1), pg.peak.astype(np.int64))
    sq = synth.bf16_bits_to_f32(pg.s)[:, None].astype(np.float64) * pg.q
    w = synth.bf16_bits_to_f32(pg.w).astype(np.float64)
    assert (np.abs(w - sq) <= 2.0 ** -8 * np.abs(sq)).all()   # half an ulp of an 8-bit significand
    again = synth.planted_groups(idx[::-7], seed=0)   # any subset, any order, same bits
    assert np.array_equal(again.w, pg.w[::-7])
    other = synth.planted_groups(idx[:100], seed=1)
    assert not np.array_equal(other.w, pg.w[:100])


def test_splitmix64_reference_values():
    # SplitMix64 seeded with 0 and stepped by its increment: the published sequence starts
    # 0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F.
    out = synth.splitmix64(np.array([0, 0x9E3779B97F4A7C15, (2 * 0x9E3779B97F4A7C15) % 2 ** 64],
                                    dtype=np.uint64))
    assert [int(v) for v in out] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_codes_and_scales_recipes():
    case = synth.case_dense_small()
    assert case.x.shape == (4, 256) and case.codes.shape == (256, 32) and case.scales.shape == (256, 8)
    s = synth.bf16_bits_to_f32(case.scales)
    assert (s >= 1e-3 * (1 - 2 ** -8)).all()
    nib = np.stack([(case.codes >> np.uint32(4 * j)) & np.uint32(0xF) for j in range(8)])
    counts = np.bincount(nib.ravel(), minlength=16)
    assert counts.min() > 0.8 * counts.mean()
