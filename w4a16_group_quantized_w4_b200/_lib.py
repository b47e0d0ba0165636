"""ctypes loader for libw4a16.so (the C ABI declared in include/w4a16.h).

The library is built in-tree by ``python -m w4a16_group_quantized_w4_b200.build``.  There is no
fallback: if the shared object is missing or does not load, every call raises.
"""
from __future__ import annotations

import ctypes as C
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libw4a16.so")

W4_OK = 0
W4_ERR_INVALID_ARG = 1
W4_ERR_UNSUPPORTED = 2
W4_ERR_CUDA = 3
W4_ERR_TIMEOUT = 4
W4_ERR_WORKSPACE = 5

W4_EPI_NONE = 0
W4_EPI_GELU_GATE = 1

W4_OP_LINEAR = 1
W4_OP_ROUTE = 2
W4_OP_GMM = 3
W4_OP_LINEAR_G = 4
W4_OP_GMM_G = 5
W4_OP_LAYER = 6
W4_OP_LAYER_CTL = 7

# name -> (restype, argtypes), mirroring include/w4a16.h
_P = C.c_void_p
_I32 = C.c_int32
_I64 = C.c_int64
_SZ = C.c_size_t
SIGNATURES = {
    "w4_repack": (_I32, [_P, _I64, _I64, _P, _P, _P, _P, _P]),
    "w4a16_linear": (_I32, [_P, _P, _P, _P, _I64, _I64, _I64, _P, _SZ, _P]),
    "moe_route_permute": (_I32, [_P, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_w4a16_gmm": (_I32, [_P, _P, _I32, _P, _P, _P, _I32, _I64, _I32, _I32, _I32, _P, _P, _SZ,
                             _P, _P]),
    "moe_combine": (_I32, [_P, _P, _P, _I32, _I32, _I32, _P, _P]),
    "w4a16_linear_noalloc": (_I32, [_P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "moe_rms_chain": (_I32, [_P, _I64, _I32, C.c_float, _P, _P]),
    "w4a16_linear_g": (_I32, [_P, _P, _P, _P, _I32, _P, _I64, _I64, _I64, _P, _SZ, _P]),
    "moe_w4a16_gmm_g": (_I32, [_P, _P, _I32, _P, _P, _P, _I32, _P, _I32, _I64, _I32, _I32, _I32, _P,
                               _P, _SZ, _P, _P]),
    "moe_w4a16_layer": (_I32, [_P, _P, _I32, _I32, _I32, _P, _P, _P, _P, _I32, _I32, _P, _P, _SZ, _P, _P]),
    "w4_workspace_bytes": (_SZ, [_I32, _I64, _I64, _I64, _I32, _I32]),
    "w4_status_str": (C.c_char_p, [_I32]),
    "w4_last_cuda_error": (_I32, []),
}

_lib = None


class W4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        lib = load()
        msg = lib.w4_status_str(status).decode()
        if status == W4_ERR_CUDA:
            msg += f" (cudaError {lib.w4_last_cuda_error()})"
        super().__init__(f"{fn} failed: {msg}")
        self.status = status


def load(path: str | None = None):
    """Load libw4a16.so once and attach the signatures.  Raises if it cannot be loaded."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(
            f"{p} is missing: build it with `python -m w4a16_group_quantized_w4_b200.build`")
    lib = C.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def check(fn: str, status: int) -> None:
    if status != W4_OK:
        raise W4Error(fn, status)
