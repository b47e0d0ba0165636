"""Seeded synthetic inputs, shared by the GPU path's tests and benchmark and by the oracle.

This module draws random numbers and stores them in the types the W4A16 path consumes: bf16
activations and scales (as uint16 bit patterns), packed int4 code words (uint32), fp32 router
logits and bf16 weights planted on the 4-bit grid.  It holds none of the method's arithmetic:
no dequantisation, no scale recovery, no routing, no matmul.  Both sides receive exactly the
arrays returned here.

Two kinds of generator live here:

* numpy ``Generator`` streams (PCG64) keyed by ``(seed, stream)`` for inputs that are built on
  the host (dense and MoE layer cases);
* a counter-based generator (SplitMix64's output function, Steele, Lea and Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014) for weights planted on the Q4_0 grid.
  Any element can be drawn from its index alone, so a GPU twin in ``csrc/synth.cu`` produces the
  same bits for full-size stacks while the host re-draws only the groups a test samples.

Workload shapes follow the synthetic stand-ins for the Gemma 4 26B-A4B mixture-of-experts layer
described in "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput",
section "The gap at 26B" (128 experts per layer, 8 active per token).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

GROUP = 32  # weights per scale along the input dimension


# --------------------------------------------------------------------------------------------
# storage-type helpers (bit patterns only)
# --------------------------------------------------------------------------------------------

def f32_to_bf16_bits(x) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest even) and return the uint16 patterns."""
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(x, dtype=np.float32)))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    """Widen bf16 patterns to float32 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(stream)])


def bf16_normal(shape, seed: int, stream: int, std: float = 1.0) -> np.ndarray:
    """bf16(N(0, std^2)) as uint16 patterns."""
    z = _rng(seed, stream).standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        z = z * np.float32(std)
    return f32_to_bf16_bits(z)


def random_code_words(shape_words, seed: int, stream: int) -> np.ndarray:
    """Uniform random uint32 words.

    A word holds eight 4-bit fields.  Uniform words make every field uniform over 0..15, i.e.
    every int4 code uniform over the 16 levels -8..7, whatever order the fields are read in.
    """
    return _rng(seed, stream).integers(0, 1 << 32, size=shape_words, dtype=np.uint64).astype(np.uint32)


def abs_normal_scales(shape, mult: float, add: float, seed: int, stream: int) -> np.ndarray:
    """bf16(mult * |N(0,1)| + add) as uint16 patterns (the configs' scale recipe)."""
    z = np.abs(_rng(seed, stream).standard_normal(shape, dtype=np.float64))
    return f32_to_bf16_bits((mult * z + add).astype(np.float32))


def zipf_bias(E: int, s: float, seed: int, stream: int) -> np.ndarray:
    """Per-expert logit bias b_e = -s * ln(rank_e), ranks a seeded permutation of 1..E.

    Adding it to N(0,1) logits makes the softmax's expert popularity follow a Zipf(s) law up to
    the noise (ln of the Zipf pmf up to a constant, which a softmax ignores).
    """
    ranks = _rng(seed, stream).permutation(E) + 1
    return (-s * np.log(ranks.astype(np.float64))).astype(np.float32)


def router_logits(T: int, E: int, seed: int, stream: int, zipf_s: float | None = None) -> np.ndarray:
    z = _rng(seed, stream).standard_normal((T, E), dtype=np.float32)
    if zipf_s is not None:
        z = (z + zipf_bias(E, zipf_s, seed, stream + 1000)[None, :]).astype(np.float32)
    return np.ascontiguousarray(z)


# --------------------------------------------------------------------------------------------
# workload cases
# --------------------------------------------------------------------------------------------

@dataclass
class DenseCase:
    """Activations x [M,K] bf16, int4 codes [N,K/8] u32 (random words), scales [N,K/32] bf16."""
    M: int
    N: int
    K: int
    x: np.ndarray
    codes: np.ndarray
    scales: np.ndarray


def dense_case(M: int, N: int, K: int, scale_mult: float, scale_add: float, seed: int = 0,
               stream0: int = 0) -> DenseCase:
    assert K % GROUP == 0
    x = bf16_normal((M, K), seed, stream0 + 1)
    codes = random_code_words((N, K // 8), seed, stream0 + 2)
    scales = abs_normal_scales((N, K // GROUP), scale_mult, scale_add, seed, stream0 + 3)
    return DenseCase(M, N, K, x, codes, scales)


@dataclass
class MoECase:
    """One mixture-of-experts layer: tokens, router logits and both expert weight stacks.

    gate/up stack: codes [E, 2I, H/8], scales [E, 2I, H/32] (rows 0..I-1 gate, I..2I-1 up);
    down stack:    codes [E, H, I/8],  scales [E, H, I/32].
    """
    T: int
    E: int
    k: int
    H: int
    I: int
    x: np.ndarray
    logits: np.ndarray
    gu_codes: np.ndarray
    gu_scales: np.ndarray
    dn_codes: np.ndarray
    dn_scales: np.ndarray


def moe_case(T: int, E: int = 128, k: int = 8, H: int = 2816, I: int = 704, seed: int = 0,
             zipf_s: float | None = None, scale_mult: float = 0.01, scale_add: float = 1e-4,
             stream0: int = 100) -> MoECase:
    assert H % GROUP == 0 and I % GROUP == 0
    x = bf16_normal((T, H), seed, stream0 + 1)
    logits = router_logits(T, E, seed, stream0 + 2, zipf_s)
    gu_codes = random_code_words((E, 2 * I, H // 8), seed, stream0 + 3)
    gu_scales = abs_normal_scales((E, 2 * I, H // GROUP), scale_mult, scale_add, seed, stream0 + 4)
    dn_codes = random_code_words((E, H, I // 8), seed, stream0 + 5)
    dn_scales = abs_normal_scales((E, H, I // GROUP), scale_mult, scale_add, seed, stream0 + 6)
    return MoECase(T, E, k, H, I, x, logits, gu_codes, gu_scales, dn_codes, dn_scales)


# The configurations the benchmark and the parity tests use.
def case_dense_small(seed: int = 0) -> DenseCase:
    """Single dense linear: x [4,256] ~ N(0,1), codes uniform, scales 0.02|N(0,1)|+1e-3."""
    return dense_case(4, 256, 256, 0.02, 1e-3, seed)


def case_dense_gemv(M: int, seed: int = 0) -> DenseCase:
    """Decode GEMV sweep point: K=4096, N=14336, scales 0.01|N(0,1)|+1e-4."""
    return dense_case(M, 14336, 4096, 0.01, 1e-4, seed)


def case_moe_decode(seed: int = 0) -> MoECase:
    """MoE decode layer: 64 tokens, 128 experts, top-8, hidden 2816, expert intermediate 704."""
    return moe_case(64, seed=seed)


ZIPF_S = 1.1


def case_moe_prefill(seed: int = 0) -> MoECase:
    """MoE prefill layer: 8192 tokens, same expert shapes, Zipf(1.1)-skewed expert popularity."""
    return moe_case(8192, seed=seed, zipf_s=ZIPF_S)


# --------------------------------------------------------------------------------------------
# counter-based planted-grid generator (host half; csrc/synth.cu is the device half)
# --------------------------------------------------------------------------------------------

_M64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB

# bf16 patterns of the scale range [1e-4, 1e-1]: bf16(1e-4) = 0x38D2, bf16(1e-1) = 0x3DCD.
SCALE_LO_BITS = 0x38D2
SCALE_HI_BITS = 0x3DCD
PLANT_ATTEMPTS = 16   # redraws of a group whose codes share a common factor
PLANT_SLOTS = 64      # counter slots per (group, attempt): 0..31 codes, 32 peak, 33 scale,
                      # 34 peak position, 35 peak sign


def splitmix64(x: np.ndarray) -> np.ndarray:
    """SplitMix64 output function applied to counters x (uint64, wrapping arithmetic)."""
    with np.errstate(over="ignore"):
        z = (np.asarray(x, dtype=np.uint64) + np.uint64(_GAMMA))
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_MIX1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_MIX2)
        return z ^ (z >> np.uint64(31))


def stream_key(seed: int, stream: int) -> int:
    return int(splitmix64(np.uint64(((int(seed) << 16) + int(stream)) & _M64)))


def _draw(key: int, ctr: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return splitmix64(np.uint64(key) + ctr.astype(np.uint64))


def _below(r: np.ndarray, n) -> np.ndarray:
    """Map 64 random bits to an integer in [0, n) via the top 32 bits (multiply-high)."""
    hi = (r >> np.uint64(32)).astype(np.uint64)
    return ((hi * np.asarray(n, dtype=np.uint64)) >> np.uint64(32)).astype(np.int64)


def _f32_bits_to_bf16_rne(b32: np.ndarray) -> np.ndarray:
    """Round finite float32 patterns to bf16 (nearest, ties to even) by integer arithmetic."""
    b = b32.astype(np.uint64)
    return ((b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)).astype(np.uint16)


@dataclass
class PlantedGroups:
    """Groups of 32 bf16 weights w_i = bf16(s * q_i) with the truth they were drawn from."""
    w: np.ndarray        # uint16 [G, 32]  bf16 weights
    q: np.ndarray        # int8   [G, 32]  planted codes (gcd of |q| is 1)
    s: np.ndarray        # uint16 [G]      planted bf16 scale
    peak: np.ndarray     # int8   [G]      planted peak level p (1..8)


def planted_groups(group_index: np.ndarray, seed: int = 0, stream: int = 500) -> PlantedGroups:
    """Draw the planted groups with the given global indices (any subset, any order).

    Per group and attempt: peak level p ~ U{1..8}; codes uniform over [-p, min(p, 7)]; one
    uniformly chosen position is set to the peak (-8 when p = 8, else +-p with a random sign);
    the scale is a bf16 pattern drawn uniformly from [bf16(1e-4), bf16(1e-1)], i.e. a uniform
    binade and a uniform mantissa (log-uniform at binade resolution).  A group whose codes share
    a factor > 1 is redrawn with the next attempt index; after the last attempt the element
    after the peak is set to 1.  Weights are bf16(s * q), the product being exact in float32.
    """
    gi = np.asarray(group_index, dtype=np.int64).ravel()
    G = gi.size
    key = stream_key(seed, stream)
    q_out = np.zeros((G, GROUP), np.int64)
    s_out = np.zeros(G, np.uint16)
    p_out = np.zeros(G, np.int64)
    todo = np.arange(G)
    slots = np.arange(GROUP, dtype=np.uint64)
    for attempt in range(PLANT_ATTEMPTS):
        if todo.size == 0:
            break
        base = ((gi[todo].astype(np.uint64) * np.uint64(PLANT_ATTEMPTS) + np.uint64(attempt))
                * np.uint64(PLANT_SLOTS))
        p = 1 + _below(_draw(key, base + np.uint64(32)), 8)
        n_s = SCALE_HI_BITS - SCALE_LO_BITS + 1
        s_bits = (SCALE_LO_BITS + _below(_draw(key, base + np.uint64(33)), n_s)).astype(np.uint16)
        pos = _below(_draw(key, base + np.uint64(34)), GROUP)
        neg = (_draw(key, base + np.uint64(35)) >> np.uint64(63)).astype(bool)
        lo = -p
        hi = np.minimum(p, 7)
        r = _draw(key, base[:, None] + slots[None, :])
        q = lo[:, None] + _below(r, (hi - lo + 1)[:, None])
        peak_val = np.where(p == 8, -8, np.where(neg, -p, p))
        q[np.arange(todo.size), pos] = peak_val
        g = np.gcd.reduce(np.abs(q), axis=1)
        ok = g == 1
        if attempt == PLANT_ATTEMPTS - 1:
            bad = ~ok
            q[np.nonzero(bad)[0], (pos[bad] + 1) % GROUP] = 1
            ok[:] = True
        idx = todo[ok]
        q_out[idx] = q[ok]
        s_out[idx] = s_bits[ok]
        p_out[idx] = p[ok]
        todo = todo[~ok]
    prod = bf16_bits_to_f32(s_out)[:, None] * q_out.astype(np.float32)  # exact
    w = _f32_bits_to_bf16_rne(prod.astype(np.float32).view(np.uint32))
    return PlantedGroups(w=w, q=q_out.astype(np.int8), s=s_out, peak=p_out.astype(np.int8))


def planted_weights(rows: int, K: int, seed: int = 0, stream: int = 500, row0: int = 0) -> PlantedGroups:
    """Planted weights for rows [row0, row0+rows) of a [*, K] matrix, groups in row-major order."""
    assert K % GROUP == 0
    gpr = K // GROUP
    idx = np.arange(row0 * gpr, (row0 + rows) * gpr, dtype=np.int64)
    return planted_groups(idx, seed, stream)


def bytes_of(*arrays) -> int:
    return int(sum(a.nbytes for a in arrays))


def log_uniform_check(s_bits: np.ndarray) -> float:
    """Fraction of scales inside [1e-4, 1e-1] (a sanity figure for the scale recipe)."""
    s = bf16_bits_to_f32(s_bits).astype(np.float64)
    return float(np.mean((s >= 1e-4 * (1 - 2 ** -8)) & (s <= 0.1 * (1 + 2 ** -8))))


__all__ = [name for name in dir() if not name.startswith("_") and name not in ("math",)]
