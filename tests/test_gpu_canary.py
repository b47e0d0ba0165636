"""Out-of-bounds writes: every output of the entry points is a window into a larger buffer whose
guard bands, before and after, hold a canary pattern; after the call the guards must be intact.

The interior results are checked elsewhere (against the oracle); here only the bytes around them
matter.  Shapes include ragged tails (N and K not multiples of the tiles, rows not multiples of
the token blocks) on both GEMM kernels, the fused layer, routing, combine and the repack.
"""
import numpy as np
import pytest
import torch

from w4a16_group_quantized_w4_b200 import api, synth
from tests._util import dev_bf16, dev_f32, dev_u32

pytestmark = pytest.mark.gpu

GUARD = 4096                      # bytes of canary on each side (a multiple of 256: alignment kept)
CANARY = 0xA5


class Guarded:
    """A tensor of `shape` and `dtype` in the middle of a byte buffer filled with CANARY."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.nbytes = n
        self.buf = torch.full((GUARD + n + GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        self.t = self.buf[GUARD:GUARD + n].view(dtype).view(*shape)

    def check(self, what):
        torch.cuda.synchronize()
        head = self.buf[:GUARD].cpu().numpy()
        tail = self.buf[GUARD + self.nbytes:].cpu().numpy()
        assert (head == CANARY).all(), f"{what}: write before the output"
        assert (tail == CANARY).all(), f"{what}: write after the output"


@pytest.mark.parametrize("M,N,K", [(3, 200, 96), (16, 330, 416), (64, 384, 512), (100, 200, 256)])
def test_linear_guards(M, N, K):
    """M < 64 takes the weight-streaming kernel, M >= 64 the tensor-core kernel when N and K fit its
    tiles (384 x 512), else streaming (200 x 256)."""
    c = synth.dense_case(M, N, K, 0.02, 1e-3, seed=M + N)
    y = Guarded((M, N), torch.bfloat16)
    api.w4a16_linear(dev_bf16(c.x), dev_u32(c.codes), dev_bf16(c.scales), y=y.t)
    y.check("w4a16_linear")
    assert torch.isfinite(y.t.float()).all()


@pytest.mark.parametrize("T,E,k,H,I", [(5, 8, 2, 96, 64), (64, 128, 8, 2816, 704), (600, 4, 2, 256, 128)])
def test_moe_calls_guards(T, E, k, H, I):
    """Routing, both grouped GEMMs (decode sizes on the streaming kernel; 600 tokens on 4 experts on
    the tensor-core kernel) and combine, every output guarded."""
    case = synth.moe_case(T, E, k, H, I, seed=T + E)
    gu_c, gu_s = dev_u32(case.gu_codes), dev_bf16(case.gu_scales)
    dn_c, dn_s = dev_u32(case.dn_codes), dev_bf16(case.dn_scales)
    ids = Guarded((T, k), torch.int32)
    w = Guarded((T, k), torch.float32)
    offs = Guarded((E + 1,), torch.int32)
    sp = Guarded((T * k,), torch.int32)
    pp = Guarded((T * k,), torch.int32)
    rt = api.Routing(ids.t, w.t, offs.t, sp.t, pp.t)
    api.moe_route_permute(dev_f32(case.logits), k, out=rt)
    for g, what in ((ids, "topk_ids"), (w, "topk_w"), (offs, "expert_offsets"), (sp, "sorted_pair"),
                    (pp, "pair_pos")):
        g.check(what)
    rows = T * k
    h = Guarded((rows, I), torch.bfloat16)
    api.moe_w4a16_gmm(dev_bf16(case.x), rt.sorted_pair, k, gu_c, gu_s, rt.expert_offsets, rows,
                      api.W4_EPI_GELU_GATE, out=h.t)
    h.check("gate/up h")
    o = Guarded((rows, H), torch.bfloat16)
    api.moe_w4a16_gmm(h.t, None, 1, dn_c, dn_s, rt.expert_offsets, rows, api.W4_EPI_NONE, out=o.t)
    o.check("down o")
    y = Guarded((T, H), torch.bfloat16)
    api.moe_combine(o.t, rt.topk_w, rt.pair_pos, y=y.t)
    y.check("combine y")
    xn = Guarded((T, H), torch.bfloat16)
    api.moe_rms_chain(y.t, x_next=xn.t)
    xn.check("rms chain")


@pytest.mark.parametrize("T", [1, 3, 64])
def test_fused_layer_guards(T):
    case = synth.moe_case(T, 128, 8, 2816, 704, seed=400 + T)
    w = (dev_u32(case.gu_codes), dev_bf16(case.gu_scales), dev_u32(case.dn_codes), dev_bf16(case.dn_scales))
    y = Guarded((T, 2816), torch.bfloat16)
    api.moe_w4a16_layer(dev_bf16(case.x), dev_f32(case.logits), 8, *w, y=y.t)
    y.check("moe_w4a16_layer y")


def test_repack_guards():
    pg = synth.planted_weights(48, 160, seed=3)
    wb = dev_bf16(pg.w.reshape(48, 160))
    codes = Guarded((48, 20), torch.int32)
    scales = Guarded((48, 5), torch.bfloat16)
    gm = Guarded((48, 5), torch.uint8)
    cnt = Guarded((1,), torch.int64)
    api.w4_repack(wb, codes=codes.t, scales=scales.t, group_m=gm.t, off_grid_count=cnt.t)
    for g, what in ((codes, "codes"), (scales, "scales"), (gm, "group_m"), (cnt, "off_grid_count")):
        g.check(what)
