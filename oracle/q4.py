"""Q4_0 grid, packed-code layout, dequantisation and scale recovery.  Test infrastructure only.

Source: "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", section
"A repack, not a re-quantization": every group of 32 weights along the input dimension sits on
a 16-level Q4_0 grid with levels -8..7; the per-group step is found by trying max|w|/m for
m = 1..8 and keeping the first step that reproduces the whole group, then refined by least
squares over the 32 values; scales are stored at bf16.  The same steps are listed in "The
Quantization Problem I Didn't Know I Had Until I Tried Running LLMs Locally", section "Building
the Missing Piece".  Dequantisation is scale times integer code, symmetric, no zero-point ("What
quantization really is", section "How the ruler works").

Readings taken where the pages are open (each is also listed in the design notes):
  * the scale is non-negative, codes lie in -8..7, so a step under which a value would need +8
    does not reproduce the group;
  * "reproduces" means: every r_i = w_i / step rounds (half to even) to an integer code in
    -8..7 and lies within 1/16 of it (bf16 storage of s*q leaves at most 7/128 of a step on a
    true grid; a wrong grid leaves at least 1/8 - 7/128);
  * "least squares over the 32 values" is the one-parameter fit min_s sum (w_i - s q_i)^2 with
    the codes fixed: s* = sum(w q) / sum(q^2), sums in index order, in float64;
  * a group that no m reproduces is "off the grid": it falls back to the textbook step
    max|w|/8 with codes clamped to -8..7, is flagged with m = 0 and counted;
  * an all-zero group has scale 0, codes 0 and m = 1; a group holding NaN or infinity is
    off the grid with codes 0 and a NaN scale.

Packed layout L1 (ours; the container's bit layout is not on the pages): codes[r, w] is a
uint32 holding u = q + 8 of elements k = 8w .. 8w+7 in k order: bits 4j..4j+3 hold element
8w + j, j = 0..7 (the lowest nibble is the lowest k).  One 16-byte run of four words is exactly
one group of 32.  Scales[r, g] is the bf16 scale of elements 32g..32g+31 of row r.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import bf16

GROUP = 32
QMIN, QMAX = -8, 7
M_MAX = 8
REPRODUCE_TOL = 1.0 / 16.0


# ------------------------------------------------------------------------------------------
# packed layout
# ------------------------------------------------------------------------------------------

def nibble_shift(j: int) -> int:
    """Bit offset of element 8w + j inside word w (layout L1: nibble j holds element j)."""
    return 4 * j


def pack(q) -> np.ndarray:
    """int codes [R, K] in -8..7 -> uint32 words [R, K/8] in the layout described above.

    Nibble j of a word at bits 4j means, in bytes: byte b of the word (bits 8b..8b+7) holds
    elements 2b (low nibble) and 2b + 1 (high nibble), and the word is read little-endian."""
    q = np.asarray(q)
    R, K = q.shape
    assert K % 8 == 0
    assert q.min(initial=0) >= QMIN and q.max(initial=0) <= QMAX
    u = (q.astype(np.int16) + 8).astype(np.uint8).reshape(R, K // 2, 2)
    byte = u[:, :, 0] | (u[:, :, 1] << np.uint8(4))
    return np.ascontiguousarray(byte).view("<u4").reshape(R, K // 8).astype(np.uint32)


def unpack(codes) -> np.ndarray:
    """uint32 words [R, K/8] -> int codes [R, K] (int64), inverse of ``pack``."""
    c = np.asarray(codes, dtype=np.uint32).astype(np.uint64)
    R, W = c.shape
    q = np.empty((R, W, 8), dtype=np.int64)
    for j in range(8):
        q[:, :, j] = ((c >> np.uint64(nibble_shift(j))) & np.uint64(0xF)).astype(np.int64) - 8
    return q.reshape(R, W * 8)


def dequant(codes, scales) -> np.ndarray:
    """W[n, k] = s[n, k // 32] * q[n, k] in float64 (exact: 8-bit times 4-bit significands).

    codes [..., N, K/8] uint32, scales [..., N, K/32] bf16 patterns -> float64 [..., N, K].
    """
    codes = np.asarray(codes)
    scales = np.asarray(scales)
    lead = codes.shape[:-1]
    q = unpack(codes.reshape(-1, codes.shape[-1]))
    s = bf16.to_f64(scales.reshape(-1, scales.shape[-1]))
    K = q.shape[1]
    assert s.shape[1] * GROUP == K
    W = q.astype(np.float64) * np.repeat(s, GROUP, axis=1)
    return W.reshape(*lead, K)


# ------------------------------------------------------------------------------------------
# scale recovery (repack)
# ------------------------------------------------------------------------------------------

@dataclass
class Repacked:
    codes: np.ndarray        # uint32 [R, K/8]
    scales: np.ndarray       # uint16 [R, K/32] bf16 patterns
    group_m: np.ndarray      # uint8  [R, K/32]: first reproducing m (1..8), 0 = off the grid
    off_grid: int            # number of groups no m reproduces
    q: np.ndarray            # int64  [R, K] the codes before packing
    s_refined: np.ndarray    # float64 [R, K/32] least-squares step before bf16 rounding


def _search_groups(w: np.ndarray):
    """Steps 1-3 of the repack for groups w [G, 32] (float64 values of bf16 weights).

    Returns (q [G, 32] int64, m [G] int64, off [G] bool, bad [G] bool).
    """
    G = w.shape[0]
    finite = np.isfinite(w).all(axis=1)
    a = np.where(finite[:, None], np.abs(w), 0.0).max(axis=1)       # step 1: a = max |w_i|
    q = np.zeros((G, GROUP), dtype=np.int64)
    m_found = np.zeros(G, dtype=np.int64)
    zero = finite & (a == 0.0)
    m_found[zero] = 1
    undecided = finite & (a > 0.0)
    for m in range(1, M_MAX + 1):                                   # step 2: m = 1, 2, ..., 8
        if not undecided.any():
            break
        idx = np.nonzero(undecided)[0]
        step = a[idx] / float(m)
        r = w[idx] / step[:, None]
        qi = np.rint(r)
        ok = ((np.abs(r - qi) <= REPRODUCE_TOL).all(axis=1)
              & (qi >= QMIN).all(axis=1) & (qi <= QMAX).all(axis=1))
        won = idx[ok]                                               # first m that reproduces
        q[won] = qi[ok].astype(np.int64)
        m_found[won] = m
        undecided[won] = False
    off = undecided                                                 # step 3: off the grid
    if off.any():
        idx = np.nonzero(off)[0]
        step8 = a[idx] / 8.0
        q[idx] = np.clip(np.rint(w[idx] / step8[:, None]), QMIN, QMAX).astype(np.int64)
        m_found[idx] = 0
    bad = ~finite
    return q, m_found, off | bad, bad


def _refine(w: np.ndarray, q: np.ndarray) -> np.ndarray:
    """Step 4: least-squares step s* = sum_i w_i q_i / sum_i q_i^2 with the codes fixed.

    Sums run in index order i = 0..31 in float64; a group whose codes are all zero gets 0.
    """
    num = np.zeros(w.shape[0], dtype=np.float64)
    den = np.zeros(w.shape[0], dtype=np.int64)
    for i in range(GROUP):
        num = num + w[:, i] * q[:, i].astype(np.float64)
        den = den + q[:, i] * q[:, i]
    s = np.zeros_like(num)
    nz = den > 0
    s[nz] = num[nz] / den[nz].astype(np.float64)
    return s


def repack(w_bits) -> Repacked:
    """Recover Q4_0 codes and bf16 scales from bf16 weights [R, K] (K % 32 == 0).

    Per group of 32 along K, in the pages' order: a = max|w|; for m = 1..8 try step a/m and keep
    the first that reproduces the group; refine the step by least squares; store it at bf16 and
    pack the codes (u = q + 8).
    """
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    R, K = w_bits.shape
    assert K % GROUP == 0
    w = bf16.to_f64(w_bits).reshape(-1, GROUP)
    q, m, off, bad = _search_groups(w)
    q[bad] = 0
    s = _refine(np.where(bad[:, None], 0.0, w), q)
    scale_bits = bf16.from_f64(s)
    scale_bits[bad] = bf16.QNAN_BITS
    s[bad] = np.nan
    qk = q.reshape(R, K)
    return Repacked(codes=pack(qk), scales=scale_bits.reshape(R, K // GROUP),
                    group_m=m.astype(np.uint8).reshape(R, K // GROUP), off_grid=int(off.sum()),
                    q=qk, s_refined=s.reshape(R, K // GROUP))


def textbook_max8(w_bits):
    """The textbook Q4_0 rule the pages warn about: step = max|w| / 8, codes clamped to -8..7.

    Returns (q [G, 32] int64, step [G] float64, reproduced [G] bool) for groups [G, 32].
    Used only to show that the rule re-rounds groups whose peak sits below level 8.
    """
    w = bf16.to_f64(np.asarray(w_bits, dtype=np.uint16)).reshape(-1, GROUP)
    a = np.abs(w).max(axis=1)
    step = a / 8.0
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(step[:, None] > 0, w / step[:, None], 0.0)
    q = np.clip(np.rint(r), QMIN, QMAX).astype(np.int64)
    reproduced = (np.abs(r - q) <= REPRODUCE_TOL).all(axis=1)
    return q, step, reproduced


def packed_bytes(rows: int, K: int) -> int:
    """Bytes of packed codes plus bf16 scales for a [rows, K] weight (4.5 bits per weight)."""
    return rows * K // 2 + rows * (K // GROUP) * 2
