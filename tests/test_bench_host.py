"""Host-side helpers of bench.py (CPU): the parity statistics of the bench line, the reading of a
committed profile summary's DRAM traffic, and the source hash that ties a summary to the kernel
source it was captured on."""
import os
import types

import numpy as np
import torch

import bench
from oracle import moe
from w4a16_group_quantized_w4_b200 import synth


def _small_ref():
    case = synth.moe_case(12, 16, 4, 256, 128, seed=11)
    ref = {}
    bench.cpu_baseline(case, ref)
    full = moe.moe_layer(case.x, case.logits, case.gu_codes, case.gu_scales, case.dn_codes, case.dn_scales,
                         case.k)
    return case, ref, full


def test_cpu_baseline_returns_its_sample():
    case, ref, full = _small_ref()
    n = ref["tokens"].size
    assert 0 < n <= case.T and np.array_equal(ref["tokens"], np.arange(n))
    np.testing.assert_allclose(ref["y"], full.y[:n], rtol=1e-12, atol=1e-15)   # (summation order)
    assert np.array_equal(ref["routing"].sorted_pair, full.routing.sorted_pair)


def test_parity_stats_within_and_outside_tolerance():
    case, ref, full = _small_ref()
    ro = full.routing
    rt = types.SimpleNamespace(topk_ids=torch.from_numpy(ro.topk_ids.astype(np.int32)),
                               expert_offsets=torch.from_numpy(ro.expert_offsets.astype(np.int32)),
                               sorted_pair=torch.from_numpy(ro.sorted_pair.astype(np.int32)),
                               pair_pos=torch.from_numpy(ro.pair_pos.astype(np.int32)))
    p = bench.parity_stats(full.y * (1 + 1e-3), ref, rt)
    n = ref["tokens"].size
    assert p["tokens_checked"] == n and p["rows_within_tolerance"] == n
    assert abs(p["max_rel_l2"] - 1e-3) < 1e-6
    assert all(p["routing_bit_exact"].values())
    # one row off by 1%: rel-L2 1e-2 > 5e-3 for that row only; a swapped permutation entry
    bad = full.y.copy()
    bad[0] *= 1.01
    sp = rt.sorted_pair.clone()
    sp[[0, 1]] = sp[[1, 0]]
    p = bench.parity_stats(bad, ref, types.SimpleNamespace(**{**vars(rt), "sorted_pair": sp}))
    assert p["rows_within_tolerance"] == n - 1
    assert p["routing_bit_exact"]["sorted_pair"] is False and p["routing_bit_exact"]["topk_ids"] is True


def test_profile_traffic_reading(tmp_path, monkeypatch):
    """A summary is read only while its recorded source hash is the current one."""
    h = bench.kernel_source_hash("stream_gemm.cu")
    assert len(h) == 16 and int(h, 16) >= 0
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "x.md").write_text(f"# t\n\n- kernel_source_sha256_16: {h}\n- dram_bytes_per_step: 1234\n")
    (prof / "y.md").write_text("# t\n\n- kernel_source_sha256_16: 0000000000000000\n- dram_bytes_per_step: 99\n")
    real_root = bench.ROOT
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the source hash still reads the real sources
    monkeypatch.setattr(bench, "kernel_source_hash", lambda src="stream_gemm.cu": h)
    assert bench.read_profile_traffic("x.md") == 1234.0
    assert bench.read_profile_traffic("y.md") is None
    assert bench.read_profile_traffic("missing.md") is None
    assert os.path.isdir(real_root)


def test_every_committed_profile_names_its_source_and_traffic():
    """Each committed ncu summary records the hash of the source it was captured on and its DRAM
    bytes, in the form bench.py reads."""
    pdir = os.path.join(bench.ROOT, "profiles")
    for name in sorted(os.listdir(pdir)):
        text = open(os.path.join(pdir, name)).read()
        assert "kernel_source_sha256_16:" in text, name
        assert "ncu " in text and "--clock-control none" in text, name
