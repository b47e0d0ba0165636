"""Pins for the oracle's Q4_0 layout, dequantisation and scale recovery (CPU only).

Method source: "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput",
section "A repack, not a re-quantization" (grid -8..7, group 32 along the input dimension, the
max/8 trap, the m-search for m = 1..8, least-squares refinement, bf16 scales, zero groups off
the grid); "The Quantization Problem I Didn't Know I Had Until I Tried Running LLMs Locally",
section "Building the Missing Piece" (the same steps).

What pins what:
  * nibble layout: the golden words in tests/golden/nibble_layout.txt and exhaustive round trip;
  * dequantisation: the closed form x = s*q, probed one weight at a time;
  * scale recovery: hand-worked groups (tests/golden/repack_groups.txt), exact recovery of
    planted codes and peaks on generated groups, the textbook rule failing below level 8,
    common-factor groups, random (off-grid) groups, and a loop-by-loop brute force.
"""
import os

import numpy as np
import pytest

from oracle import bf16, q4
from w4a16_group_quantized_w4_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_blocks(path):
    blocks, cur = [], None
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.partition(" ")
        if key == "name":
            cur = {"name": rest}
            blocks.append(cur)
        else:
            cur[key] = rest
    return blocks


def test_page_constants():
    const = {}
    for line in open(os.path.join(GOLDEN, "page_constants.txt")):
        if line.startswith("#") or not line.strip():
            continue
        name, value = line.split("|")[0].split()
        const[name] = value
    assert int(const["group_size"]) == q4.GROUP
    assert (q4.QMIN, q4.QMAX) == (int(const["level_min"]), int(const["level_max"]))
    assert q4.QMAX - q4.QMIN + 1 == int(const["grid_levels"])
    assert q4.M_MAX == int(const["m_max"])


def test_nibble_layout_golden():
    for line in open(os.path.join(GOLDEN, "nibble_layout.txt")):
        if line.startswith("#") or not line.strip():
            continue
        lhs, rhs = line.split("->")
        q = np.array([int(v) for v in lhs.split()], dtype=np.int64)[None, :]
        word = int(rhs.strip(), 16)
        assert q4.pack(q)[0, 0] == word
        assert np.array_equal(q4.unpack(np.array([[word]], dtype=np.uint32))[0], q[0])


def test_pack_roundtrip_every_level_every_position():
    for pos in range(8):
        for level in range(-8, 8):
            q = np.zeros((1, 16), dtype=np.int64)
            q[0, pos] = level
            q[0, 8 + pos] = -level - 1
            assert np.array_equal(q4.unpack(q4.pack(q)), q)
    rng = np.random.default_rng(3)
    q = rng.integers(-8, 8, size=(7, 96))
    assert np.array_equal(q4.unpack(q4.pack(q)), q)


def test_dequant_is_scale_times_code_probe_by_probe():
    rng = np.random.default_rng(4)
    q = rng.integers(-8, 8, size=(5, 64))
    s_bits = synth.f32_to_bf16_bits(rng.uniform(0.01, 1.0, size=(5, 2)).astype(np.float32))
    W = q4.dequant(q4.pack(q), s_bits)
    s = bf16.to_f64(s_bits)
    for n in range(5):
        for k in range(64):
            assert W[n, k] == s[n, k // 32] * float(q[n, k])


@pytest.mark.parametrize("block", _read_blocks(os.path.join(GOLDEN, "repack_groups.txt")),
                         ids=lambda b: b["name"])
def test_repack_hand_worked_groups(block):
    w = np.array([int(v, 16) for v in block["w"].split()], dtype=np.uint16)[None, :]
    res = q4.repack(w)
    assert int(res.group_m[0, 0]) == int(block["expect_m"])
    assert int(res.scales[0, 0]) == int(block["expect_scale"], 16)
    assert np.array_equal(res.q[0], np.array([int(v) for v in block["expect_q"].split()]))
    assert res.off_grid == (1 if int(block["expect_m"]) == 0 else 0)
    _, _, reproduced = q4.textbook_max8(w)
    assert bool(reproduced[0]) == bool(int(block["textbook_reproduces"]))


def test_repack_recovers_planted_codes_exactly():
    pg = synth.planted_groups(np.arange(40_000), seed=0)
    res = q4.repack(pg.w.reshape(-1, 64))
    q = res.q.reshape(-1, 32)
    assert np.array_equal(q, pg.q.astype(np.int64))           # bit-exact codes
    assert res.off_grid == 0                                   # zero groups off the grid
    assert np.array_equal(res.group_m.reshape(-1), pg.peak.astype(np.uint8))
    s_match = np.mean(res.scales.reshape(-1) == pg.s)
    assert s_match >= 0.99, s_match
    # reported analogue of the pages' fidelity figures (bit-identical share, worst rel. diff)
    w_back = bf16.from_f64(bf16.to_f64(res.scales.reshape(-1))[:, None] * q)
    ident = np.mean(w_back == pg.w)
    w0 = bf16.to_f64(pg.w)
    w1 = bf16.to_f64(w_back)
    nz = w0 != 0
    worst = np.max(np.abs(w1[nz] - w0[nz]) / np.abs(w0[nz]))
    assert ident > 0.99 and worst < 2e-2, (ident, worst)


def test_textbook_rule_fails_when_peak_below_eight():
    pg = synth.planted_groups(np.arange(20_000), seed=1)
    q, step, reproduced = q4.textbook_max8(pg.w)
    below = np.isin(pg.peak, [3, 5, 6, 7])
    assert below.sum() > 1000
    assert not reproduced[below].any()
    assert reproduced[pg.peak == 8].all()
    w = bf16.to_f64(pg.w)
    err = np.abs(step[:, None] * q - w)
    rel = np.linalg.norm(err, axis=1) / np.linalg.norm(w, axis=1)
    # the pages report about 5% median error per group on real weights; planted data is similar
    assert 0.01 < np.median(rel[below]) < 0.2


def test_common_factor_group_recovers_reduced_codes():
    rng = np.random.default_rng(7)
    for g in (2, 3, 4):
        for _ in range(20):
            p = g * rng.integers(1, 8 // g + 1)           # planted peak level, a multiple of g
            hi = min(p // g, 7 // g)                       # keep every code g*base within -8..7
            base = rng.integers(-(p // g), hi + 1, size=32)
            base[rng.integers(32)] = -(p // g)             # the peak sits at -p
            s = 2.0 ** -rng.integers(3, 12)
            w = bf16.from_f64(s * g * base)[None, :]
            res = q4.repack(w)
            m = int(res.group_m[0, 0])
            assert m >= 1
            k = (p // g) // m
            assert k * m == p // g
            assert np.array_equal(res.q[0] * k, base)


def test_random_normal_groups_are_off_grid():
    rng = np.random.default_rng(8)
    w = synth.f32_to_bf16_bits(rng.standard_normal((2000, 32)).astype(np.float32))
    res = q4.repack(w)
    assert res.off_grid >= 1990
    assert (res.q >= -8).all() and (res.q <= 7).all()


def test_non_finite_group_is_flagged():
    w = np.zeros((1, 64), dtype=np.uint16)
    w[0, 3] = 0x7FC0
    w[0, 40] = 0x3F80
    res = q4.repack(w)
    assert res.off_grid == 1
    assert res.group_m[0, 0] == 0 and res.scales[0, 0] == 0x7FC0
    assert (res.q[0, :32] == 0).all()
    assert res.group_m[0, 1] == 1 and res.scales[0, 1] == 0x3F80 and res.q[0, 40] == 1


def _brute_group(wv):
    """Loop-by-loop restatement of the rule for one group of Python floats."""
    if any(v != v or v in (float("inf"), float("-inf")) for v in wv):
        return [0] * 32, 0
    a = max(abs(v) for v in wv)
    if a == 0.0:
        return [0] * 32, 1
    for m in range(1, 9):
        step = a / m
        codes = []
        good = True
        for v in wv:
            r = v / step
            c = round(r)                      # Python rounds half to even
            if abs(r - c) > 1 / 16 or c < -8 or c > 7:
                good = False
                break
            codes.append(c)
        if good:
            return codes, m
    step = a / 8
    return [min(7, max(-8, round(v / step))) for v in wv], 0


def test_brute_force_small_mixture():
    rng = np.random.default_rng(9)
    planted = synth.planted_groups(np.arange(300), seed=2).w
    normal = synth.f32_to_bf16_bits(rng.standard_normal((100, 32)).astype(np.float32))
    ties = synth.f32_to_bf16_bits((rng.integers(-16, 17, size=(50, 32)) / 2.0).astype(np.float32))
    w = np.concatenate([planted, normal, ties])
    res = q4.repack(w)
    wf = bf16.to_f64(w)
    for g in range(w.shape[0]):
        codes, m = _brute_group([float(v) for v in wf[g]])
        assert res.q[g].tolist() == codes, g
        assert int(res.group_m[g, 0]) == m
        num = 0.0
        for v, c in zip(wf[g], codes):
            num += float(v) * c
        den = sum(c * c for c in codes)
        s = num / den if den else 0.0
        assert int(res.scales[g, 0]) == int(bf16.from_f64(np.array([s]))[0])


def test_packed_bytes_four_and_a_half_bits():
    # int4 codes plus one bf16 scale per 32 weights: 4 + 16/32 = 4.5 bits per weight
    assert q4.packed_bytes(1408, 2816) * 8 == 1408 * 2816 * 4.5
