"""PyTorch-facing binding of libw4a16: one function per C entry point, same names.

Argument marshalling only: shapes, dtypes and devices are checked, outputs are allocated with
torch when the caller does not pass them, and the C function runs on the current (or given)
CUDA stream.  Every step of the computation happens in the library's kernels.

Tensor conventions: bf16 values travel as ``torch.bfloat16`` tensors, packed int4 words as
``torch.int32`` tensors holding the uint32 bit patterns (layout L1, see include/w4a16.h).
"""
from __future__ import annotations

import ctypes as C

import torch

from . import _lib

W4_EPI_NONE = _lib.W4_EPI_NONE
W4_EPI_GELU_GATE = _lib.W4_EPI_GELU_GATE


def _p(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _s(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _need(name, t, dtype, shape=None, dev=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if dev is not None and t.device != dev:
        raise ValueError(f"{name}: expected device {dev}, got {t.device}")


_WS: dict = {}


def workspace(nbytes: int, device, stream=None) -> torch.Tensor | None:
    """A scratch buffer of at least nbytes for calls on (device, stream).

    One buffer per stream: calls on one stream run in order, so they may share it (the library
    clears what it relies on, so contents left by earlier calls do not matter), while calls on
    different streams never do.  A buffer that is outgrown is kept alive, not freed, so a CUDA
    graph captured with it stays valid; a capture on its own stream gets its own buffer.
    """
    if nbytes == 0:
        return None
    dev = torch.device(device)
    if dev.index is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    key = (dev, s.cuda_stream)
    bufs = _WS.setdefault(key, [])
    if not bufs or bufs[-1].numel() < nbytes:
        bufs.append(torch.zeros((nbytes + 255) // 256 * 256, dtype=torch.uint8, device=dev))
    return bufs[-1]


def w4_workspace_bytes(op: int, m_or_t: int, n: int, k_dim: int, e: int, k: int) -> int:
    return int(_lib.load().w4_workspace_bytes(op, m_or_t, n, k_dim, e, k))


def w4_repack(w, codes=None, scales=None, group_m=None, off_grid_count=None, stream=None):
    """bf16 weights [rows, K] -> (codes int32 [rows, K/8], scales bf16 [rows, K/32],
    group_m uint8 [rows, K/32], off_grid_count int64 [1])."""
    lib = _lib.load()
    rows, K = w.shape
    _need("w", w, torch.bfloat16)
    dev = w.device
    codes = torch.empty((rows, K // 8), dtype=torch.int32, device=dev) if codes is None else codes
    scales = torch.empty((rows, K // 32), dtype=torch.bfloat16, device=dev) if scales is None else scales
    group_m = torch.empty((rows, K // 32), dtype=torch.uint8, device=dev) if group_m is None else group_m
    if off_grid_count is None:
        off_grid_count = torch.empty(1, dtype=torch.int64, device=dev)
    _need("codes", codes, torch.int32, (rows, K // 8), dev)
    _need("scales", scales, torch.bfloat16, (rows, K // 32), dev)
    _need("group_m", group_m, torch.uint8, (rows, K // 32), dev)
    _need("off_grid_count", off_grid_count, torch.int64, (1,), dev)
    _lib.check("w4_repack", lib.w4_repack(_p(w), rows, K, _p(codes), _p(scales), _p(group_m),
                                          _p(off_grid_count), _s(stream)))
    return codes, scales, group_m, off_grid_count


def w4a16_linear(x, codes, scales, y=None, ws=None, stream=None):
    """y [M, N] = x [M, K] @ dequant(codes, scales)^T, bf16 out."""
    lib = _lib.load()
    M, K = x.shape
    N = codes.shape[0]
    dev = x.device
    _need("x", x, torch.bfloat16)
    _need("codes", codes, torch.int32, (N, K // 8), dev)
    _need("scales", scales, torch.bfloat16, (N, K // 32), dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if y is None else y
    _need("y", y, torch.bfloat16, (M, N), dev)
    nbytes = w4_workspace_bytes(_lib.W4_OP_LINEAR, M, N, K, 1, 1)
    if ws is None:
        ws = workspace(nbytes, dev, stream)
    _lib.check("w4a16_linear", lib.w4a16_linear(_p(x), _p(codes), _p(scales), _p(y), M, N, K,
                                                _p(ws), 0 if ws is None else ws.numel(), _s(stream)))
    return y


def w4a16_linear_g(x, codes, scales, group: int, zeros=None, y=None, ws=None, stream=None):
    """The linear on the weight-format variants: scales [N, K/group] bf16, zeros [N, K/group]
    uint8 zero-points (or None: z = 8); W = s * (u - z)."""
    lib = _lib.load()
    M, K = x.shape
    N = codes.shape[0]
    dev = x.device
    _need("x", x, torch.bfloat16)
    _need("codes", codes, torch.int32, (N, K // 8), dev)
    _need("scales", scales, torch.bfloat16, (N, K // group), dev)
    if zeros is not None:
        _need("zeros", zeros, torch.uint8, (N, K // group), dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if y is None else y
    _need("y", y, torch.bfloat16, (M, N), dev)
    if ws is None:
        ws = workspace(w4_workspace_bytes(_lib.W4_OP_LINEAR_G, M, N, K, 1, 1), dev, stream)
    _lib.check("w4a16_linear_g", lib.w4a16_linear_g(_p(x), _p(codes), _p(scales), _p(zeros), group, _p(y),
                                                    M, N, K, _p(ws), 0 if ws is None else ws.numel(),
                                                    _s(stream)))
    return y


NOALLOC_SCRATCH_BYTES = 8 << 20


def w4a16_linear_noalloc(x, codes, scales, y=None, stream=None):
    """Like w4a16_linear, but never needs a workspace: split-K scratch comes from the library's
    fixed 8 MiB device array (for callers that cannot allocate device memory).  Calls that
    overlap on the GPU share that array and must be ordered by the caller."""
    lib = _lib.load()
    M, K = x.shape
    N = codes.shape[0]
    dev = x.device
    _need("x", x, torch.bfloat16)
    _need("codes", codes, torch.int32, (N, K // 8), dev)
    _need("scales", scales, torch.bfloat16, (N, K // 32), dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if y is None else y
    _need("y", y, torch.bfloat16, (M, N), dev)
    _lib.check("w4a16_linear_noalloc", lib.w4a16_linear_noalloc(_p(x), _p(codes), _p(scales), _p(y),
                                                                M, N, K, _s(stream)))
    return y


class Routing:
    __slots__ = ("topk_ids", "topk_w", "expert_offsets", "sorted_pair", "pair_pos")

    def __init__(self, topk_ids, topk_w, expert_offsets, sorted_pair, pair_pos):
        self.topk_ids = topk_ids
        self.topk_w = topk_w
        self.expert_offsets = expert_offsets
        self.sorted_pair = sorted_pair
        self.pair_pos = pair_pos


def moe_route_permute(logits, k: int, out: Routing | None = None, ws=None, stream=None) -> Routing:
    """Top-k routing of float32 logits [T, E] and the expert-major permutation."""
    lib = _lib.load()
    T, E = logits.shape
    dev = logits.device
    _need("logits", logits, torch.float32)
    if out is None:
        out = Routing(torch.empty((T, k), dtype=torch.int32, device=dev),
                      torch.empty((T, k), dtype=torch.float32, device=dev),
                      torch.empty(E + 1, dtype=torch.int32, device=dev),
                      torch.empty(T * k, dtype=torch.int32, device=dev),
                      torch.empty(T * k, dtype=torch.int32, device=dev))
    _need("topk_ids", out.topk_ids, torch.int32, (T, k), dev)
    _need("topk_w", out.topk_w, torch.float32, (T, k), dev)
    _need("expert_offsets", out.expert_offsets, torch.int32, (E + 1,), dev)
    _need("sorted_pair", out.sorted_pair, torch.int32, (T * k,), dev)
    _need("pair_pos", out.pair_pos, torch.int32, (T * k,), dev)
    nbytes = w4_workspace_bytes(_lib.W4_OP_ROUTE, T, 0, 0, E, k)
    if ws is None:
        ws = workspace(nbytes, dev, stream)
    _lib.check("moe_route_permute", lib.moe_route_permute(
        _p(logits), T, E, k, _p(out.topk_ids), _p(out.topk_w), _p(out.expert_offsets),
        _p(out.sorted_pair), _p(out.pair_pos), _p(ws), 0 if ws is None else ws.numel(), _s(stream)))
    return out


def moe_w4a16_gmm(a, a_row_of_pair, k: int, codes, scales, expert_offsets, rows: int,
                  epilogue: int = W4_EPI_NONE, out=None, ws=None, dev_status=None, stream=None):
    """Grouped W4A16 GEMM: codes [E, N, K/8], scales [E, N, K/32]; out [rows, N or N/2] bf16."""
    lib = _lib.load()
    E, N, Kw = codes.shape
    K = Kw * 8
    dev = a.device
    _need("a", a, torch.bfloat16)
    if a.shape[1] != K:
        raise ValueError("a: wrong number of columns")
    if a_row_of_pair is not None:
        _need("a_row_of_pair", a_row_of_pair, torch.int32, (rows,), dev)
    _need("codes", codes, torch.int32, (E, N, K // 8), dev)
    _need("scales", scales, torch.bfloat16, (E, N, K // 32), dev)
    _need("expert_offsets", expert_offsets, torch.int32, (E + 1,), dev)
    n_out = N // 2 if epilogue == W4_EPI_GELU_GATE else N
    out = torch.empty((rows, n_out), dtype=torch.bfloat16, device=dev) if out is None else out
    _need("out", out, torch.bfloat16, (rows, n_out), dev)
    nbytes = w4_workspace_bytes(_lib.W4_OP_GMM, rows, N, K, E, k)
    if ws is None:
        ws = workspace(nbytes, dev, stream)
    if dev_status is not None:
        _need("dev_status", dev_status, torch.int32, (1,), dev)
    _lib.check("moe_w4a16_gmm", lib.moe_w4a16_gmm(
        _p(a), _p(a_row_of_pair), k, _p(codes), _p(scales), _p(expert_offsets), E, rows, N, K,
        epilogue, _p(out), _p(ws), 0 if ws is None else ws.numel(), _p(dev_status), _s(stream)))
    return out


def moe_combine(o, topk_w, pair_pos, y=None, stream=None):
    """y [T, H] = sum_j topk_w[t, j] * o[pair_pos[t*k + j]] (bf16 out)."""
    lib = _lib.load()
    T, k = topk_w.shape
    H = o.shape[1]
    dev = o.device
    _need("o", o, torch.bfloat16, (T * k, H), dev)
    _need("topk_w", topk_w, torch.float32, (T, k), dev)
    _need("pair_pos", pair_pos, torch.int32, (T * k,), dev)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if y is None else y
    _need("y", y, torch.bfloat16, (T, H), dev)
    _lib.check("moe_combine", lib.moe_combine(_p(o), _p(topk_w), _p(pair_pos), T, k, H, _p(y),
                                              _s(stream)))
    return y


RMS_EPS = 1e-6


def moe_rms_chain(y, x_next=None, eps: float = RMS_EPS, stream=None):
    """x_next [T, H] = bf16(y / sqrt(mean over each row of y^2 + eps)): the input of the next
    layer of a stack (bf16 in and out)."""
    lib = _lib.load()
    T, H = y.shape
    dev = y.device
    _need("y", y, torch.bfloat16, (T, H), dev)
    x_next = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if x_next is None else x_next
    _need("x_next", x_next, torch.bfloat16, (T, H), dev)
    _lib.check("moe_rms_chain", lib.moe_rms_chain(_p(y), T, H, eps, _p(x_next), _s(stream)))
    return x_next


def moe_w4a16_gmm_g(a, a_row_of_pair, k: int, codes, scales, expert_offsets, rows: int, group: int,
                    zeros=None, epilogue: int = W4_EPI_NONE, out=None, ws=None, dev_status=None,
                    stream=None):
    """The grouped GEMM on the weight-format variants: scales [E, N, K/group], zeros
    [E, N, K/group] uint8 or None."""
    lib = _lib.load()
    E, N, Kw = codes.shape
    K = Kw * 8
    dev = a.device
    _need("a", a, torch.bfloat16)
    if a.shape[1] != K:
        raise ValueError("a: wrong number of columns")
    if a_row_of_pair is not None:
        _need("a_row_of_pair", a_row_of_pair, torch.int32, (rows,), dev)
    _need("codes", codes, torch.int32, (E, N, K // 8), dev)
    _need("scales", scales, torch.bfloat16, (E, N, K // group), dev)
    if zeros is not None:
        _need("zeros", zeros, torch.uint8, (E, N, K // group), dev)
    _need("expert_offsets", expert_offsets, torch.int32, (E + 1,), dev)
    n_out = N // 2 if epilogue == W4_EPI_GELU_GATE else N
    out = torch.empty((rows, n_out), dtype=torch.bfloat16, device=dev) if out is None else out
    _need("out", out, torch.bfloat16, (rows, n_out), dev)
    if ws is None:
        ws = workspace(w4_workspace_bytes(_lib.W4_OP_GMM_G, rows, N, K, E, k), dev, stream)
    if dev_status is not None:
        _need("dev_status", dev_status, torch.int32, (1,), dev)
    _lib.check("moe_w4a16_gmm_g", lib.moe_w4a16_gmm_g(
        _p(a), _p(a_row_of_pair), k, _p(codes), _p(scales), _p(zeros), group, _p(expert_offsets), E,
        rows, N, K, epilogue, _p(out), _p(ws), 0 if ws is None else ws.numel(), _p(dev_status),
        _s(stream)))
    return out


def moe_layer_fusable(T: int, E: int, k: int, H: int, I: int) -> bool:
    """Whether moe_w4a16_layer accepts these sizes (1 <= T <= 128, T k <= 6 E, E <= 576)."""
    return T >= 1 and w4_workspace_bytes(_lib.W4_OP_LAYER, T, H, I, E, k) > 0


def layer_workspace(T: int, E: int, k: int, H: int, I: int, device) -> torch.Tensor:
    """A private workspace for moe_w4a16_layer, zero-filled (its control area must start at
    zero; every call leaves it so).  Not shared with other calls."""
    nbytes = w4_workspace_bytes(_lib.W4_OP_LAYER, T, H, I, E, k)
    if nbytes == 0:
        raise _lib.W4Error("moe_w4a16_layer", _lib.W4_ERR_UNSUPPORTED)
    return torch.zeros((nbytes + 255) // 256 * 256, dtype=torch.uint8, device=device)


def moe_w4a16_layer(x, logits, k: int, gu_codes, gu_scales, dn_codes, dn_scales, y=None, ws=None,
                    dev_status=None, stream=None):
    """One MoE decode layer in one kernel launch: x bf16 [T, H], logits f32 [T, E], gate/up
    codes [E, 2I, H/8] / scales [E, 2I, H/32], down codes [E, H, I/8] / scales [E, H, I/32]
    -> y bf16 [T, H].  ws: a workspace from layer_workspace (allocated here when None)."""
    lib = _lib.load()
    T, H = x.shape
    E, N2, _ = gu_codes.shape
    I = N2 // 2
    dev = x.device
    _need("x", x, torch.bfloat16, (T, H), dev)
    _need("logits", logits, torch.float32, (T, E), dev)
    _need("gu_codes", gu_codes, torch.int32, (E, 2 * I, H // 8), dev)
    _need("gu_scales", gu_scales, torch.bfloat16, (E, 2 * I, H // 32), dev)
    _need("dn_codes", dn_codes, torch.int32, (E, H, I // 8), dev)
    _need("dn_scales", dn_scales, torch.bfloat16, (E, H, I // 32), dev)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if y is None else y
    _need("y", y, torch.bfloat16, (T, H), dev)
    if ws is None:
        ws = layer_workspace(T, E, k, H, I, dev)
    _need("ws", ws, torch.uint8, None, dev)
    if dev_status is not None:
        _need("dev_status", dev_status, torch.int32, (1,), dev)
    _lib.check("moe_w4a16_layer", lib.moe_w4a16_layer(
        _p(x), _p(logits), T, E, k, _p(gu_codes), _p(gu_scales), _p(dn_codes), _p(dn_scales), H, I,
        _p(y), _p(ws), ws.numel(), _p(dev_status), _s(stream)))
    return y


class MoELayer:
    """One mixture-of-experts layer on the device: the four entry points composed on one stream
    (route -> gate/up GEMM with the GELU gate -> down GEMM -> combine), with every buffer
    allocated once so that a step launches kernels only.  fused=True runs the same layer as one
    moe_w4a16_layer launch (decode sizes only; its routing, h and o then stay in the layer's
    private workspace)."""

    def __init__(self, gu_codes, gu_scales, dn_codes, dn_scales, T: int, k: int, fused: bool = False):
        self.E, self.N2, _ = gu_codes.shape
        self.H = gu_codes.shape[2] * 8
        self.I = self.N2 // 2
        self.T, self.k = T, k
        dev = gu_codes.device
        self.w = (gu_codes, gu_scales, dn_codes, dn_scales)
        self.fused = fused
        if fused:
            self.layer_ws = layer_workspace(T, self.E, k, self.H, self.I, dev)
            self.y = torch.empty((T, self.H), dtype=torch.bfloat16, device=dev)
            return
        self.rt = Routing(torch.empty((T, k), dtype=torch.int32, device=dev),
                          torch.empty((T, k), dtype=torch.float32, device=dev),
                          torch.empty(self.E + 1, dtype=torch.int32, device=dev),
                          torch.empty(T * k, dtype=torch.int32, device=dev),
                          torch.empty(T * k, dtype=torch.int32, device=dev))
        self.h = torch.empty((T * k, self.I), dtype=torch.bfloat16, device=dev)
        self.o = torch.empty((T * k, self.H), dtype=torch.bfloat16, device=dev)
        self.y = torch.empty((T, self.H), dtype=torch.bfloat16, device=dev)
        nr = w4_workspace_bytes(_lib.W4_OP_ROUTE, T, 0, 0, self.E, k)
        # private: the routing outputs of layers that run back to back must not share scratch
        self.route_ws = torch.zeros(nr, dtype=torch.uint8, device=dev) if nr else None

    def __call__(self, x, logits, stream=None):
        gu_c, gu_s, dn_c, dn_s = self.w
        if self.fused:
            return moe_w4a16_layer(x, logits, self.k, gu_c, gu_s, dn_c, dn_s, y=self.y,
                                   ws=self.layer_ws, stream=stream)
        moe_route_permute(logits, self.k, out=self.rt, ws=self.route_ws, stream=stream)
        moe_w4a16_gmm(x, self.rt.sorted_pair, self.k, gu_c, gu_s, self.rt.expert_offsets,
                      self.T * self.k, W4_EPI_GELU_GATE, out=self.h, stream=stream)
        moe_w4a16_gmm(self.h, None, 1, dn_c, dn_s, self.rt.expert_offsets, self.T * self.k,
                      W4_EPI_NONE, out=self.o, stream=stream)
        moe_combine(self.o, self.rt.topk_w, self.rt.pair_pos, y=self.y, stream=stream)
        return self.y
