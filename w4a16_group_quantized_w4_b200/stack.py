"""A stack of mixture-of-experts layers held on one device.

The whole-model form of the hot path: every layer's gate/up and down weights arrive as bf16 (the
"unquantized" QAT export of "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8
throughput", section "A repack, not a re-quantization"), are repacked on the device by
`w4_repack` into int4 codes and bf16 scales, and decode steps then run the four entry points layer
after layer ("The gap at 26B": 128 experts per layer, 8 active).  The pages give no blocks
between the MoE layers; a chained step feeds each layer the previous layer's output divided by
its root mean square (moe_rms_chain, no learned weight), with seeded router logits per layer.

Layouts (layer-major, so layer l's weights are contiguous slices):
  gate/up codes [L, E, 2I, H/8] int32, scales [L, E, 2I, H/32] bf16
  down    codes [L, E, H, I/8]  int32, scales [L, E, H, I/32]  bf16
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import api


@dataclass
class RepackReport:
    off_grid_gate_up: int
    off_grid_down: int
    group_m_gate_up: torch.Tensor     # uint8 [L*E*2I, H/32]
    group_m_down: torch.Tensor        # uint8 [L*E*H, I/32]


class MoEStack:
    """L layers of E experts (hidden H, expert intermediate I, top-k routing) on one device."""

    def __init__(self, L: int, E: int = 128, k: int = 8, H: int = 2816, I: int = 704, device="cuda"):
        self.L, self.E, self.k, self.H, self.I = L, E, k, H, I
        dev = torch.device(device)
        self.gu_codes = torch.empty((L, E, 2 * I, H // 8), dtype=torch.int32, device=dev)
        self.gu_scales = torch.empty((L, E, 2 * I, H // 32), dtype=torch.bfloat16, device=dev)
        self.dn_codes = torch.empty((L, E, H, I // 8), dtype=torch.int32, device=dev)
        self.dn_scales = torch.empty((L, E, H, I // 32), dtype=torch.bfloat16, device=dev)
        self._layers = {}

    # ------------------------------------------------------------------ repack
    def gate_up_rows(self) -> int:
        return self.L * self.E * 2 * self.I

    def down_rows(self) -> int:
        return self.L * self.E * self.H

    def repack(self, w_gate_up: torch.Tensor, w_down: torch.Tensor, stream=None) -> RepackReport:
        """w_gate_up bf16 [L*E*2I, H], w_down bf16 [L*E*H, I] (layer-major) -> this stack's codes
        and scales, through two w4_repack calls."""
        dev = self.gu_codes.device
        g_gu = torch.empty((self.gate_up_rows(), self.H // 32), dtype=torch.uint8, device=dev)
        g_dn = torch.empty((self.down_rows(), self.I // 32), dtype=torch.uint8, device=dev)
        off = torch.zeros(2, dtype=torch.int64, device=dev)
        api.w4_repack(w_gate_up, codes=self.gu_codes.view(-1, self.H // 8),
                      scales=self.gu_scales.view(-1, self.H // 32), group_m=g_gu,
                      off_grid_count=off[0:1], stream=stream)
        api.w4_repack(w_down, codes=self.dn_codes.view(-1, self.I // 8),
                      scales=self.dn_scales.view(-1, self.I // 32), group_m=g_dn,
                      off_grid_count=off[1:2], stream=stream)
        o = off.cpu()
        return RepackReport(int(o[0]), int(o[1]), g_gu, g_dn)

    # ------------------------------------------------------------------ decode
    def fusable(self, T: int) -> bool:
        """Whether T tokens fit the single-launch fused layer (moe_w4a16_layer)."""
        return api.moe_layer_fusable(T, self.E, self.k, self.H, self.I)

    def layer(self, l: int, T: int, fused: bool = False) -> api.MoELayer:
        """MoE layer l for T tokens (buffers allocated once per (l, T, fused)): the four-call
        path, or the single-launch fused layer when fused and T fits it."""
        fused = fused and self.fusable(T)
        key = (l, T, fused)
        if key not in self._layers:
            self._layers[key] = api.MoELayer(self.gu_codes[l], self.gu_scales[l], self.dn_codes[l],
                                             self.dn_scales[l], T, self.k, fused=fused)
        return self._layers[key]

    def step(self, xs, logits, stream=None, fused: bool = False):
        """One decode step through every layer with independent inputs: xs[l] bf16 [T, H],
        logits[l] f32 [T, E] -> the list of layer outputs y_l bf16 [T, H] (each layer's own
        buffer)."""
        T = xs[0].shape[0]
        return [self.layer(l, T, fused)(xs[l], logits[l], stream=stream) for l in range(self.L)]

    def chained_step(self, x0, logits, stream=None, fused: bool = False):
        """One decode step through the chained stack: layer 0 takes x0 bf16 [T, H]; layer l + 1
        takes moe_rms_chain(y_l).  Returns (the inputs x_l, the outputs y_l), device buffers
        owned by the stack (overwritten by the next chained step of the same T and path)."""
        T = x0.shape[0]
        key = ("chain", T, fused)
        if key not in self._layers:
            self._layers[key] = [torch.empty((T, self.H), dtype=torch.bfloat16, device=x0.device)
                                 for _ in range(self.L - 1)]
        xb = self._layers[key]
        xs, ys = [x0], []
        for l in range(self.L):
            y = self.layer(l, T, fused)(xs[l], logits[l], stream=stream)
            ys.append(y)
            if l + 1 < self.L:
                xs.append(api.moe_rms_chain(y, x_next=xb[l], stream=stream))
        return xs, ys

    def expert_bytes(self) -> int:
        """Packed bytes of one expert (gate/up + down codes and scales)."""
        return (2 * self.I * self.H // 2 + 2 * self.I * self.H // 16 +
                self.H * self.I // 2 + self.H * self.I // 16)
