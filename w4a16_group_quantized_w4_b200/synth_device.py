"""Device twin of the planted-weight generator (libw4synth.so).

`planted(ngroups, group0, seed, stream)` draws the same groups as `synth.planted_groups` (same
counter-based SplitMix64 recipe, bit for bit) directly into device memory, for workloads too large
to generate on the host (30 layers x 128 experts of bf16 weights).  Input generation only: the
library under test is never called from here.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libw4synth.so")
_LIB = None


def load():
    global _LIB
    if _LIB is None:
        if not os.path.exists(_PATH):
            raise RuntimeError(f"{_PATH} is missing: run `python -m w4a16_group_quantized_w4_b200.build`")
        lib = C.CDLL(_PATH)
        lib.w4s_planted.restype = C.c_int
        lib.w4s_planted.argtypes = [C.c_uint64, C.c_uint32, C.c_int64, C.c_int64, C.c_void_p,
                                    C.c_void_p, C.c_void_p, C.c_void_p]
        lib.w4s_code_mismatches.restype = C.c_int
        lib.w4s_code_mismatches.argtypes = [C.c_uint64, C.c_uint32, C.c_int64, C.c_int64, C.c_void_p,
                                            C.c_void_p, C.c_void_p]
        _LIB = lib
    return _LIB


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def planted(ngroups: int, group0: int = 0, seed: int = 0, stream: int = 500, w=None,
            with_truth: bool = False, device="cuda"):
    """bf16 weights [ngroups * 32] of planted groups group0 .. group0 + ngroups - 1 (and, with
    with_truth, the planted codes int8 [ngroups, 32] and scale bits int16 [ngroups])."""
    lib = load()
    if w is None:
        w = torch.empty(ngroups * 32, dtype=torch.bfloat16, device=device)
    assert w.numel() == ngroups * 32 and w.is_contiguous() and w.data_ptr() % 16 == 0
    q = torch.empty((ngroups, 32), dtype=torch.int8, device=device) if with_truth else None
    s = torch.empty(ngroups, dtype=torch.int16, device=device) if with_truth else None
    st = torch.cuda.current_stream(w.device).cuda_stream
    rc = lib.w4s_planted(seed, stream, group0, ngroups, _ptr(w), _ptr(q), _ptr(s), C.c_void_p(st))
    if rc != 0:
        raise RuntimeError(f"w4s_planted failed: cudaError {rc}")
    return (w, q, s) if with_truth else w


def code_mismatches(codes, group0: int, ngroups: int, seed: int = 0, stream: int = 500) -> int:
    """Number of groups whose packed codes (4 int32 words per group, layout L1) differ from the
    planted codes of groups group0 .. group0 + ngroups - 1."""
    lib = load()
    assert codes.is_contiguous() and codes.numel() >= ngroups * 4
    cnt = torch.zeros(1, dtype=torch.int64, device=codes.device)
    st = torch.cuda.current_stream(codes.device).cuda_stream
    rc = lib.w4s_code_mismatches(seed, stream, group0, ngroups, _ptr(codes), _ptr(cnt), C.c_void_p(st))
    if rc != 0:
        raise RuntimeError(f"w4s_code_mismatches failed: cudaError {rc}")
    return int(cnt.item())
