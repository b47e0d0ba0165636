"""The arithmetic identities the weight-streaming kernel relies on, checked on the CPU in numpy
(a model of the method, independent of the kernel and of the oracle).

Per group of 32 along K the kernel multiplies exact biased codes by fp16 activations and removes
the bias with one per-group correction (the C operand of the group's first MMA):
  even nibble positions: (1024 + u) * x'            - 1032 * x'       = (u - 8) * x'
  odd nibble positions:  (1024 + 16 u) * (x' / 16)  - 1152 * (x' / 16) = (u - 8) * x'
so d = sum (u - 8) x' exactly in exact arithmetic; with float32 sums, the error stays within a few
float32 units of the bias term, far inside the bf16 rounding of an output.  x' = fp16(x * 2^f)
with f putting the row's largest |x| in [2^14, 2^15).
"""
import numpy as np


def _row_exponent(x):
    m = np.abs(x).max()
    return 14 - int(np.floor(np.log2(m)))          # largest |x| * 2^f in [2^14, 2^15)


def _group(rng, scale=1.0):
    x = (rng.standard_normal(32) * scale).astype(np.float32)
    u = rng.integers(0, 16, size=32)
    return x, u


def test_biased_codes_and_correction_cancel_exactly():
    """With exact (float64) sums the correction leaves exactly sum (u - 8) x'."""
    rng = np.random.default_rng(0)
    for _ in range(200):
        x, u = _group(rng)
        f = _row_exponent(x)
        xp = (x.astype(np.float64) * 2.0 ** f).astype(np.float16).astype(np.float64)
        even = np.arange(32) % 8 < 4              # (any fixed split of the 32 positions works)
        a = np.where(even, xp, 0.0)
        b = np.where(even, 0.0, (xp / 16).astype(np.float16).astype(np.float64))
        w_even = 1024.0 + u
        w_odd = 1024.0 + 16.0 * u
        c = -(1032.0 * a.sum() + 1152.0 * b.sum())
        d = c + (w_even * a).sum() + (w_odd * b).sum()
        want = ((u - 8) * np.where(even, xp, b * 16)).sum()
        assert d == want


def test_biased_products_are_exact_in_fp16_and_float32():
    """1024 + u and 1024 + 16 u are exact fp16 values, and their products with fp16 activations
    are exact in float32 (11-bit significands)."""
    u = np.arange(16)
    assert np.array_equal((1024.0 + u).astype(np.float16).astype(np.float64), 1024.0 + u)
    assert np.array_equal((1024.0 + 16 * u).astype(np.float16).astype(np.float64), 1024.0 + 16 * u)
    rng = np.random.default_rng(1)
    x = rng.standard_normal(10000).astype(np.float16)
    for w in (1024.0, 1039.0, 1024.0 + 16 * 15):
        p32 = np.float32(w) * x.astype(np.float32)
        assert np.array_equal(p32.astype(np.float64), w * x.astype(np.float64))


def test_float32_group_sum_error_bound():
    """Summing the 32 biased products and the correction in float32 (any order) stays within
    32 float32 units of the bias term (2^-24 * 1152 * 2^15 each), which relative to an output's
    bf16 rounding (2^-9) is negligible."""
    rng = np.random.default_rng(2)
    worst = 0.0
    for _ in range(300):
        x, u = _group(rng, scale=rng.uniform(0.01, 10))
        f = _row_exponent(x)
        xp = (x.astype(np.float64) * 2.0 ** f).astype(np.float16).astype(np.float32)
        even = np.arange(32) % 8 < 4
        a = np.where(even, xp, np.float32(0))
        b = np.where(even, np.float32(0), (xp / np.float32(16)).astype(np.float16).astype(np.float32))
        w = np.where(even, np.float32(1024) + u.astype(np.float32), np.float32(1024) + 16 * u.astype(np.float32))
        v = np.where(even, a, b)
        c = np.float32(-(np.float32(1032) * a.sum(dtype=np.float32) + np.float32(1152) * b.sum(dtype=np.float32)))
        order = rng.permutation(32)
        d = c
        for i in order:
            d = np.float32(d + w[i] * v[i])
        exact = ((u - 8) * np.where(even, a.astype(np.float64), b.astype(np.float64) * 16)).sum()
        bound = 32 * 2.0 ** -24 * 1152 * 2.0 ** 15 * 2
        assert abs(float(d) - exact) <= bound
        worst = max(worst, abs(float(d) - exact) / bound)
    assert worst < 1.0
