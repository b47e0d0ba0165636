"""Helpers shared by the tests: host<->device moves of raw bit patterns and the row tolerance."""
from __future__ import annotations

import numpy as np
import torch

# Float tolerance for the bf16-output GEMMs, per output row (token):
# relative L2 error <= 5e-3 and max abs error <= 2e-2 * max|y_ref|, against the float64 oracle.
REL_L2 = 5e-3
MAX_ABS_FRAC = 2e-2


def dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def dev_u32(words: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(words).view(np.int32)).to(device)


def dev_f32(x: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def host_bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def host_u32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy().view(np.uint32)


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_rows_close(y: np.ndarray, ref: np.ndarray, rel_l2=REL_L2, max_abs_frac=MAX_ABS_FRAC,
                      what="y"):
    y = np.asarray(y, dtype=np.float64).reshape(ref.shape[0], -1)
    ref = np.asarray(ref, dtype=np.float64).reshape(ref.shape[0], -1)
    assert np.isfinite(y).all(), f"{what}: non-finite output"
    err = y - ref
    nref = np.linalg.norm(ref, axis=1)
    nerr = np.linalg.norm(err, axis=1)
    mref = np.abs(ref).max(axis=1)
    merr = np.abs(err).max(axis=1)
    zero = nref == 0
    assert (nerr[zero] == 0).all(), f"{what}: rows with zero reference are not zero"
    rel = np.where(zero, 0.0, nerr / np.where(zero, 1, nref))
    bad = np.nonzero((rel > rel_l2) | (merr > max_abs_frac * mref))[0]
    assert bad.size == 0, (f"{what}: {bad.size} rows out of tolerance, worst rel-L2 "
                           f"{rel.max():.3e}, row {bad[:5]}")
    return float(rel.max())
