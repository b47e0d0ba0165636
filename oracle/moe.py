"""Mixture-of-experts W4A16 layer: routing, permutation, grouped expert GEMMs, combine.

Test infrastructure only.

Sources:
  * "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", section "The
    gap at 26B" (128 experts per layer, 8 active per token) and section "What changed in vLLM's
    TPU backend" (the experts' packed int4 weights and 32-wide scales go to a grouped matmul
    that dequantises each weight tile before the multiply; activations stay bf16);
  * "What quantization really is", section "Gemma 4 puts numbers on the tip" (all experts stay
    loaded; about 4B of the 26B parameters are active per token).

Readings taken where the pages are silent (router math, gate/up split, activation, combine are
not on the pages):
  * routing: the k largest fp32 logits per token, ties broken towards the lower expert index,
    listed in descending order; weights are the softmax over the selected k logits (equal to
    the full softmax renormalised over them), evaluated in float64;
  * permutation: pairs p = t*k + j are ordered by (expert, p) ascending (a stable counting
    sort); ``expert_offsets`` is the exclusive prefix sum of the per-expert counts and
    ``pair_pos`` the inverse permutation;
  * the gate/up weight has 2I rows: rows 0..I-1 are the gate, rows I..2I-1 the up projection;
    h = gelu_tanh(gate) * up with gelu_tanh(z) = z/2 * (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3)));
  * combine: y[t] = sum over slots j = 0..k-1 of w[t, j] * o[pair_pos[t*k + j]];
  * chaining of stacked layers (the pages give no blocks between the MoE layers, and the gated
    expert MLP is quadratic in its input, so plain chaining grows without bound): the next
    layer's input is the output divided by its root mean square, with no learned weight,
    x_next = bf16(y / sqrt(mean(y^2) + eps)), eps = 1e-6.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

from . import bf16, q4

EPI_NONE = 0
EPI_GELU_GATE = 1


@dataclass
class Routing:
    topk_ids: np.ndarray       # int32 [T, k]
    topk_w: np.ndarray         # float64 [T, k]
    counts: np.ndarray         # int64 [E]
    expert_offsets: np.ndarray  # int32 [E + 1]
    sorted_pair: np.ndarray    # int32 [T * k]
    pair_pos: np.ndarray       # int32 [T * k]


def route(logits, k: int) -> Routing:
    """Top-k of E router logits per token, softmax weights over the selected, stable permutation."""
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    assert 1 <= k <= E
    l = logits.astype(np.float64)
    order = np.argsort(-l, axis=1, kind="stable")   # descending logit, equal logits by index
    ids = order[:, :k]
    sel = np.take_along_axis(l, ids, axis=1)
    e = np.exp(sel - sel[:, :1])                     # sel[:, 0] is the largest selected logit
    w = e / e.sum(axis=1, keepdims=True)
    flat = ids.reshape(-1)
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    sorted_pair = np.argsort(flat, kind="stable")    # by (expert, pair index)
    pair_pos = np.empty_like(sorted_pair)
    pair_pos[sorted_pair] = np.arange(T * k)
    return Routing(ids.astype(np.int32), w, counts, offsets.astype(np.int32),
                   sorted_pair.astype(np.int32), pair_pos.astype(np.int32))


def gelu_tanh(z) -> np.ndarray:
    """GELU, tanh form: z/2 * (1 + tanh(sqrt(2/pi) * (z + 0.044715 z^3))), float64."""
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3)))


def gmm(a_bits, a_row_of_pair, k: int, codes, scales, expert_offsets, epilogue: int,
        rows=None) -> np.ndarray:
    """Grouped W4A16 GEMM over experts, float64, one output row per routed pair (sorted order).

    a_bits [A, K] bf16 activations; for sorted row r of expert e (off[e] <= r < off[e+1]) the
    input row is a[a_row_of_pair[r] // k] when ``a_row_of_pair`` is given (gather of token rows),
    else a[r].  codes [E, N, K/8], scales [E, N, K/32].  Output row r = input row times
    W_e^T ([N] values), or, with the GELU gate, gelu_tanh(first N/2) * (last N/2).
    ``rows`` restricts the evaluation to the listed sorted rows (others are NaN).
    """
    a = bf16.to_f64(np.asarray(a_bits, dtype=np.uint16))
    codes = np.asarray(codes)
    scales = np.asarray(scales)
    off = np.asarray(expert_offsets, dtype=np.int64)
    E, N = codes.shape[0], codes.shape[1]
    n_rows = int(off[-1])
    N_out = N // 2 if epilogue == EPI_GELU_GATE else N
    out = np.full((n_rows, N_out), np.nan)
    want = np.ones(n_rows, bool) if rows is None else np.isin(np.arange(n_rows), rows)
    for e in range(E):
        r = np.arange(off[e], off[e + 1])
        r = r[want[r]]
        if r.size == 0:
            continue
        src = (np.asarray(a_row_of_pair)[r] // k) if a_row_of_pair is not None else r
        W = q4.dequant(codes[e], scales[e])          # [N, K]
        Y = a[src] @ W.T
        if epilogue == EPI_GELU_GATE:
            I = N // 2
            Y = gelu_tanh(Y[:, :I]) * Y[:, I:]
        out[r] = Y
    return out


def combine(o, topk_w, pair_pos, T: int, k: int) -> np.ndarray:
    """y[t] = sum_{j=0..k-1} w[t, j] * o[pair_pos[t*k + j]], float64, slots in order."""
    o = np.asarray(o, dtype=np.float64)
    w = np.asarray(topk_w, dtype=np.float64).reshape(T, k)
    pp = np.asarray(pair_pos).reshape(T, k)
    y = np.zeros((T, o.shape[1]))
    for j in range(k):
        y = y + w[:, j:j + 1] * o[pp[:, j]]
    return y


@dataclass
class LayerResult:
    y: np.ndarray          # float64 [T, H] (rows not evaluated are NaN)
    h: np.ndarray          # float64 [T*k, I] sorted order
    o: np.ndarray          # float64 [T*k, H] sorted order
    routing: Routing


def moe_layer(x_bits, logits, gu_codes, gu_scales, dn_codes, dn_scales, k: int,
              tokens=None, h_bf16: bool = False) -> LayerResult:
    """One MoE layer: route -> gate/up GEMM + GELU gate -> down GEMM -> weighted combine.

    ``tokens`` restricts evaluation to those token indices.  ``h_bf16`` rounds the
    intermediate h to bf16 (mirrors a bf16 intermediate; reported, not a parity reading).
    """
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    T = x_bits.shape[0]
    rt = route(logits, k)
    rows = None
    if tokens is not None:
        tokens = np.asarray(tokens, dtype=np.int64)
        rows = rt.pair_pos.reshape(T, k)[tokens].reshape(-1)
    h = gmm(x_bits, rt.sorted_pair, k, gu_codes, gu_scales, rt.expert_offsets, EPI_GELU_GATE, rows)
    if h_bf16:
        h = bf16.to_f64(bf16.from_f64(h))
    n_rows = h.shape[0]
    o = np.full((n_rows, np.asarray(dn_codes).shape[1]), np.nan)
    off = rt.expert_offsets.astype(np.int64)
    want = np.ones(n_rows, bool) if rows is None else np.isin(np.arange(n_rows), rows)
    for e in range(off.size - 1):
        r = np.arange(off[e], off[e + 1])
        r = r[want[r]]
        if r.size == 0:
            continue
        W = q4.dequant(np.asarray(dn_codes)[e], np.asarray(dn_scales)[e])
        o[r] = h[r] @ W.T  # the down GEMM consumes h in float64
    if tokens is None:
        y = combine(o, rt.topk_w, rt.pair_pos, T, k)
    else:
        y = np.full((T, o.shape[1]), np.nan)
        pp = rt.pair_pos.reshape(T, k)
        acc = np.zeros((tokens.size, o.shape[1]))
        for j in range(k):
            acc = acc + rt.topk_w[tokens, j:j + 1] * o[pp[tokens, j]]
        y[tokens] = acc
    return LayerResult(y=y, h=h, o=o, routing=rt)


RMS_EPS = 1e-6


def rms_chain(y_bits, eps: float = RMS_EPS) -> np.ndarray:
    """Next layer's input from a layer's output: bf16(y / sqrt(mean over the row of y^2 + eps)),
    per row, float64 then rounded to nearest even (bf16 bit patterns in and out)."""
    y = bf16.to_f64(np.asarray(y_bits, dtype=np.uint16))
    r = np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + eps)
    return bf16.from_f64(y / r)
