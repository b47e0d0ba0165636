"""The C-ABI library loads and exports every entry point include/w4a16.h declares (CPU only).

Also checks host-side argument validation, which returns before any CUDA call.
"""
import ctypes as C
import os
import re

import pytest

from w4a16_group_quantized_w4_b200 import _lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "w4a16.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("w4_repack", "w4a16_linear", "moe_route_permute", "moe_w4a16_gmm", "moe_combine",
                 "w4_workspace_bytes", "w4_status_str", "w4_last_cuda_error"):
        assert must in names


def test_every_declared_symbol_is_exported():
    lib = _lib.load()
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) <= set(_lib.SIGNATURES)


def test_host_validation_rejects_bad_arguments():
    lib = _lib.load()
    nul = C.c_void_p(None)
    bogus = C.c_void_p(16)
    assert lib.w4_repack(bogus, 4, 33, bogus, bogus, nul, nul, nul) == _lib.W4_ERR_INVALID_ARG
    assert lib.w4_repack(nul, 4, 64, bogus, bogus, nul, nul, nul) == _lib.W4_ERR_INVALID_ARG
    assert lib.w4a16_linear(bogus, bogus, bogus, bogus, 1, 0, 64, nul, 0, nul) == _lib.W4_ERR_INVALID_ARG
    assert lib.w4a16_linear(C.c_void_p(18), bogus, bogus, bogus, 1, 8, 64, nul, 0, nul) == _lib.W4_ERR_INVALID_ARG
    assert lib.moe_route_permute(bogus, 4, 128, 0, bogus, bogus, bogus, bogus, bogus, nul, 0, nul) == _lib.W4_ERR_INVALID_ARG
    assert lib.moe_route_permute(bogus, 4, 2000, 8, bogus, bogus, bogus, bogus, bogus, nul, 0, nul) == _lib.W4_ERR_INVALID_ARG
    assert lib.moe_w4a16_gmm(bogus, nul, 1, bogus, bogus, bogus, 8, 16, 63, 64, 1, bogus, nul, 0, nul, nul) == _lib.W4_ERR_INVALID_ARG
    assert lib.moe_w4a16_gmm(bogus, nul, 1, bogus, bogus, bogus, 8, 16, 64, 64, 7, bogus, nul, 0, nul, nul) == _lib.W4_ERR_INVALID_ARG
    assert lib.moe_combine(bogus, bogus, bogus, 4, 8, 12, bogus, nul) == _lib.W4_ERR_INVALID_ARG
    assert lib.w4_status_str(_lib.W4_ERR_TIMEOUT) == b"W4_ERR_TIMEOUT"
    assert lib.w4_workspace_bytes(99, 1, 1, 32, 1, 1) == 0


def test_fused_layer_sizes_and_range():
    """moe_w4a16_layer's workspace sizing and its range checks (both before any CUDA call)."""
    lib = _lib.load()
    nul = C.c_void_p(None)
    bogus = C.c_void_p(256)
    ws = lib.w4_workspace_bytes(_lib.W4_OP_LAYER, 64, 2816, 704, 128, 8)
    ctl = lib.w4_workspace_bytes(_lib.W4_OP_LAYER_CTL, 0, 2816, 704, 128, 8)
    # the control area does not depend on T, and sits inside every T's workspace
    assert ctl == lib.w4_workspace_bytes(_lib.W4_OP_LAYER_CTL, 64, 2816, 704, 128, 8)
    assert 0 < ctl < lib.w4_workspace_bytes(_lib.W4_OP_LAYER, 1, 2816, 704, 128, 8) < ws
    # h and o alone: 512 rows of 704 and 2816 bf16
    assert ws > 512 * (704 + 2816) * 2
    assert lib.w4_workspace_bytes(_lib.W4_OP_LAYER, 129, 2816, 704, 128, 8) == 0   # T > 128
    assert lib.w4_workspace_bytes(_lib.W4_OP_LAYER, 97, 2816, 704, 128, 8) == 0    # T k > 6 E
    assert lib.w4_workspace_bytes(_lib.W4_OP_LAYER, 96, 2816, 704, 128, 8) > ws
    args = (bogus, bogus, bogus, bogus, 2816, 704, bogus, bogus, 1 << 30, nul, nul)
    assert lib.moe_w4a16_layer(bogus, bogus, 129, 128, 8, *args) == _lib.W4_ERR_UNSUPPORTED
    assert lib.moe_w4a16_layer(bogus, bogus, 97, 128, 8, *args) == _lib.W4_ERR_UNSUPPORTED
    assert lib.moe_w4a16_layer(bogus, bogus, 4, 1024, 8, *args) == _lib.W4_ERR_UNSUPPORTED   # E > 576
    assert lib.moe_w4a16_layer(bogus, bogus, 4, 128, 0, *args) == _lib.W4_ERR_INVALID_ARG
    bad_h = (bogus, bogus, bogus, bogus, 2800, 704, bogus, bogus, 1 << 30, nul, nul)
    assert lib.moe_w4a16_layer(bogus, bogus, 4, 128, 8, *bad_h) == _lib.W4_ERR_INVALID_ARG
    assert lib.moe_w4a16_layer(nul, bogus, 4, 128, 8, *args) == _lib.W4_ERR_INVALID_ARG
    assert lib.moe_w4a16_layer(nul, nul, 0, 128, 8, *args) == _lib.W4_OK      # nothing to do


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError):
        _lib.load(str(tmp_path / "nope.so"))


def test_binding_signatures_match_the_header():
    """The ctypes argument lists in _lib.SIGNATURES have the arity and the integer widths of the
    declarations in include/w4a16.h (a drifted binding would pass arguments in the wrong slots)."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    decls = dict(re.findall(r"\b([A-Za-z_][A-Za-z0-9_]*)\s*\(([^;{}]*?)\)\s*;", text, flags=re.S))
    width = {"int32_t": C.c_int32, "int64_t": C.c_int64, "size_t": C.c_size_t, "float": C.c_float}
    for name, (_, args) in _lib.SIGNATURES.items():
        assert name in decls, name
        params = [p.strip() for p in decls[name].replace("\n", " ").split(",") if p.strip() and p.strip() != "void"]
        assert len(params) == len(args), (name, len(params), len(args))
        for p, a in zip(params, args):
            if "*" in p:
                assert a is C.c_void_p, (name, p)
                continue
            base = p.replace("const", "").split()[0]
            if base in width:
                assert a is width[base], (name, p, a)
