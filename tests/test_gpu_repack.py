"""GPU parity of w4_repack against the oracle: bit-exact codes, scales, group_m and off-grid count.

Method: "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput", section
"A repack, not a re-quantization" (m-search for m = 1..8, least-squares refinement, bf16 scale,
zero groups off the grid on QAT data).
"""
import os

import numpy as np
import pytest
import torch

from oracle import bf16, q4
from w4a16_group_quantized_w4_b200 import api, synth
from tests._util import dev_bf16, host_bf16_bits, host_u32

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _gpu_repack(w_bits: np.ndarray):
    w = dev_bf16(w_bits)
    codes, scales, gm, cnt = api.w4_repack(w)
    torch.cuda.synchronize()
    return host_u32(codes), host_bf16_bits(scales), gm.cpu().numpy(), int(cnt.item())


def _check(w_bits: np.ndarray):
    ref = q4.repack(w_bits)
    codes, scales, gm, cnt = _gpu_repack(w_bits)
    assert np.array_equal(codes, ref.codes), "codes differ"
    assert np.array_equal(scales, ref.scales), "scales differ"
    assert np.array_equal(gm, ref.group_m), "group_m differs"
    assert cnt == ref.off_grid
    return ref


def test_planted_groups_bit_exact():
    pg = synth.planted_groups(np.arange(64 * 1000), seed=3)
    ref = _check(pg.w.reshape(-1, 256))
    assert ref.off_grid == 0


def test_random_and_tie_groups_bit_exact():
    rng = np.random.default_rng(5)
    normal = synth.f32_to_bf16_bits(rng.standard_normal((500, 32)).astype(np.float32))
    ties = synth.f32_to_bf16_bits((rng.integers(-16, 17, size=(500, 32)) / 2.0).astype(np.float32))
    small = synth.f32_to_bf16_bits((rng.standard_normal((200, 32)) * 1e-38).astype(np.float32))
    huge = synth.f32_to_bf16_bits((rng.standard_normal((200, 32)) * 1e36).astype(np.float32))
    _check(np.concatenate([normal, ties, small, huge]).reshape(-1, 64))


def test_golden_and_crafted_groups():
    blocks = []
    for line in open(os.path.join(GOLDEN, "repack_groups.txt")):
        if line.startswith("w "):
            blocks.append([int(v, 16) for v in line.split()[1:]])
    g = np.array(blocks, dtype=np.uint16)
    # least-squares step exactly on a bf16 midpoint: w = (1, 1 + 2^-7) -> s* = 1 + 2^-8 -> 1.0
    mid = np.zeros((1, 32), np.uint16)
    mid[0, 0] = 0x3F80
    mid[0, 1] = 0x3F81
    nan = np.zeros((1, 32), np.uint16)
    nan[0, 7] = 0x7FC0
    inf = np.zeros((1, 32), np.uint16)
    inf[0, 9] = 0xFF80
    sub = np.zeros((1, 32), np.uint16)
    sub[0, :4] = [0x0001, 0x0002, 0x8003, 0x0004]        # subnormal bf16 values
    negz = np.full((1, 32), 0x8000, np.uint16)
    ref = _check(np.concatenate([g, mid, nan, inf, sub, negz]))
    assert ref.scales[len(blocks), 0] == 0x3F80


@pytest.mark.parametrize("rows,K", [(1, 32), (3, 96), (7, 2816), (129, 704)])
def test_ragged_shapes(rows, K):
    pg = synth.planted_weights(rows, K, seed=11)
    _check(pg.w.reshape(rows, K))


def test_expert_stack_slice():
    """A slice of a planted expert stack (gate/up rows of 2816 inputs), as the model layout."""
    pg = synth.planted_weights(1408, 2816, seed=0)
    ref = _check(pg.w.reshape(1408, 2816))
    assert ref.off_grid == 0
    assert np.array_equal(ref.q.reshape(-1, 32), pg.q.astype(np.int64))
