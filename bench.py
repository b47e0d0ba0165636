#!/usr/bin/env python
"""Benchmark of the W4A16 group-32 mixture-of-experts layer on B200.

Default workload: one MoE decode layer with 64 tokens, 128 experts, top-8 routing, hidden 2816,
expert intermediate 704 (gate/up int4 [128, 1408, 2816], down int4 [128, 2816, 704], group 32,
bf16 scales).  A step is one pass of the hot path: route + permute, gate/up grouped GEMM with the
GELU gate, down grouped GEMM, weighted combine.  Metric: tokens per second (higher is better).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                  [--workload moe_decode|moe_prefill] [--no-secondary] [--stack-layers L]

Multi-GPU: the layer does not shard; N ranks run N independent replicas (weak scaling, no
data-path collective), timed on the device with the max over ranks.  `--impl reference` times the CPU oracle
(the correctness reference) on the same workload, one token per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE W4A16 grouped-GEMM tokens/s; achieved HBM GB/s / TC util vs B200 peak"
UNIT = "tokens/s"

WORKLOADS = {
    "moe_decode": dict(T=64, zipf=None, name="moe_decode_T64_E128_top8_H2816_I704_g32"),
    "moe_prefill": dict(T=8192, zipf=1.1, name="moe_prefill_T8192_E128_top8_H2816_I704_g32_zipf1.1"),
    # the dense decode GEMV of the sweep (a separate line for profiling; not the headline)
    "dense_gemv": dict(T=16, zipf=None, name="dense_gemv_M16_K4096_N14336_g32"),
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=list(WORKLOADS), default="moe_decode")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--stack-layers", type=int, default=30,
                    help="layers of the secondary repack + expert-stack measurement (30: the full stack)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--path", choices=["four_call", "fused"], default="four_call",
                    help="decode layer as four calls (six kernels) or as the single-launch fused layer")
    return ap.parse_args()


# ------------------------------------------------------------------------------------------
# distributed plumbing
# ------------------------------------------------------------------------------------------

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def ranks_init(world, backend="nccl", device=None, timeout_s=120):
    """Join the job's process group (one process per GPU, env:// rendezvous as torchrun sets it
    up), with a short timeout so that ranks waiting on a lost peer end with an error."""
    if world <= 1:
        return
    import torch.distributed as dist
    from datetime import timedelta
    kw = {"timeout": timedelta(seconds=timeout_s)}
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def ranks_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def ranks_max(x, world, device=None):
    """The maximum of x over all ranks: a job's device time is its slowest rank's."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, ms):
    """Whole-job units per second: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / (ms / 1e3)


def ranks_finish(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu_index), "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which):
        if which == "begin":
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        time.sleep(0.25)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            rows.append((ts, parts))
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        inside = [r for r in rows if self.t0 is not None and self.t0 - 0.15 <= r[0] <= (self.t1 or r[0]) + 0.15]
        use = inside if inside else rows
        sm = [float(p[1]) for _, p in use if p[1].replace(".", "").isdigit()]
        smax = [float(p[2]) for _, p in use if p[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for _, p in use:
            for name, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(use),
                "power_w_max": max((float(p[3]) for _, p in use if p[3].replace(".", "").isdigit()), default=None)}


# ------------------------------------------------------------------------------------------
# native arm
# ------------------------------------------------------------------------------------------

def to_dev(a, kind, device):
    import numpy as np
    import torch
    if kind == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    if kind == "u32":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).to(device)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def gmm_bytes(counts, T, k, H, I):
    """Algorithmic bytes of the two grouped GEMM launches: codes + scales of every expert that
    received a token, activations read once, outputs written once."""
    hit = int((counts > 0).sum())
    gu_w = 2 * I * (H // 8) * 4 + 2 * I * (H // 32) * 2
    dn_w = H * (I // 8) * 4 + H * (I // 32) * 2
    gu = hit * gu_w + T * H * 2 + T * k * I * 2
    dn = hit * dn_w + T * k * I * 2 + T * k * H * 2
    return gu, dn, hit


# the sources a kernel is compiled from (the kernel's file, the headers holding its device code)
KERNEL_SOURCES = {
    "stream_gemm.cu": ["stream_gemm.cu", "stream_gemm.cuh", "common.cuh"],
    "fused.cu": ["fused.cu", "stream_gemm.cuh", "route.cuh", "common.cuh"],
}


def kernel_source_hash(src="stream_gemm.cu"):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(src, [src]):
        h.update(open(os.path.join(ROOT, "w4a16_group_quantized_w4_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def read_profile_traffic(name, src="stream_gemm.cu", key="dram_bytes_per_step"):
    """DRAM bytes of one step's grouped-GEMM launches from a committed ncu summary, if taken on
    the current kernel source (None otherwise)."""
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if ":" in line and line.strip().startswith("- "):
            k, _, v = line.strip()[2:].partition(":")
            vals[k.strip()] = v.strip()
    if vals.get("kernel_source_sha256_16") != kernel_source_hash(src):
        return None
    try:
        return float(vals[key])
    except (KeyError, ValueError):
        return None


def native_gemv(args, world, rank, local):
    """The dense GEMV (M = 16, K = 4096, N = 14336) as its own line: w4a16_linear calls replayed
    from CUDA graphs over 8 rotating weight copies (264 MB, more than twice L2)."""
    import torch

    from w4a16_group_quantized_w4_b200 import api, synth

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    ranks_init(world, "nccl", device)
    M, K, N, nc = WORKLOADS["dense_gemv"]["T"], 4096, 14336, 8
    base = synth.case_dense_gemv(M, seed=args.seed + rank)
    codes = [to_dev(base.codes, "u32", device) for _ in range(nc)]
    scales = [to_dev(base.scales, "bf16", device) for _ in range(nc)]
    x = to_dev(base.x, "bf16", device)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            api.w4a16_linear(x, codes[i % nc], scales[i % nc], y=y)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(nc):
                api.w4a16_linear(x, codes[i], scales[i], y=y)
        g.replay()
    stream.synchronize()
    reps = max(1, args.steps // nc)
    ranks_barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    stream.synchronize()
    ms = ranks_max(e0.elapsed_time(e1), world, device)
    calls = reps * nc
    us = ms * 1e3 / calls
    hbm_peak, _, _, peak_src = peaks()
    byts = N * K // 2 + N * (K // 32) * 2 + M * K * 2 + M * N * 2
    del g
    ranks_finish(world)
    if rank != 0:
        return
    print(json.dumps({
        "metric": "dense W4A16 GEMV rows/s", "value": round(job_throughput(M * calls, world, ms), 1),
        "unit": "rows/s", "n_gpus": world, "steps": calls, "warmup": args.warmup, "ms_per_step": round(us / 1e3, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded: codes uniform over -8..7, scales 0.01|N(0,1)|+1e-4, x N(0,1))",
        "config": {"workload": WORKLOADS["dense_gemv"]["name"], "M": M, "K": K, "N": N,
                   "l2": f"no flush: {nc} weight copies (264 MB) rotate"},
        "gpu_launches": 2 * calls,
        "roofline": {"bound": "hbm", "achieved": round(byts / us / 1e3, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(byts / us / 1e3 / hbm_peak, 4),
                     "traffic": read_profile_traffic("stream_gemm_dense_gemv.md", key="dram_bytes_per_call"),
                     "kernel": "stream_gemm_kernel with its preparation pass", "algorithmic_bytes_per_call": byts,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"},
    }), flush=True)


def native(args, world, rank, local):
    import numpy as np
    import torch

    from w4a16_group_quantized_w4_b200 import api, synth

    if args.workload == "dense_gemv":
        return native_gemv(args, world, rank, local)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    ranks_init(world, "nccl", device)
    wl = WORKLOADS[args.workload]
    T, E, k, H, I = wl["T"], 128, 8, 2816, 704
    case = synth.moe_case(T, E, k, H, I, seed=args.seed + rank, zipf_s=wl["zipf"])
    fused = args.path == "fused"
    if fused and not api.moe_layer_fusable(T, E, k, H, I):
        raise SystemExit(f"--path fused: {wl['name']} is outside the fused layer's range")
    copies = 2
    layers = []
    for c in range(copies):
        layers.append(api.MoELayer(to_dev(case.gu_codes, "u32", device), to_dev(case.gu_scales, "bf16", device),
                                   to_dev(case.dn_codes, "u32", device), to_dev(case.dn_scales, "bf16", device), T, k,
                                   fused=fused))
    x = to_dev(case.x, "bf16", device)
    logits = to_dev(case.logits, "f32", device)
    stream = torch.cuda.Stream(device)
    torch.cuda.synchronize()

    # warm-up, then capture consecutive steps into a CUDA graph
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            layers[i % copies](x, logits)
    stream.synchronize()
    # one graph holds `spg` consecutive steps (alternating the weight copies), as a model's
    # forward pass would capture its layers together; the timed region replays it steps / spg times
    spg = 10 if args.steps % 10 == 0 else (2 if args.steps % 2 == 0 else 1)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(spg):
            layers[i % copies](x, logits)
    with torch.cuda.stream(stream):
        for i in range(3):
            graph.replay()
    stream.synchronize()

    # ---------------- timed region (device step, graph replay) ----------------
    gpu_index = _physical_gpu_index(local)
    clocks = ClockSampler(gpu_index)
    clocks.start()
    ranks_barrier(world)
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    clocks.mark("begin")
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for i in range(args.steps // spg):
            graph.replay()
        ev1.record(stream)
    stream.synchronize()
    clocks.mark("end")
    torch.cuda.synchronize()
    ms = ranks_max(ev0.elapsed_time(ev1), world, device)
    ranks_barrier(world)
    clocks.stop()
    ms_per_step = ms / args.steps
    value = job_throughput(T * args.steps, world, ms)

    # distribution of the step time: 100 graph replays, each between its own events
    dist = []
    with torch.cuda.stream(stream):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(100)]
        for a, b in evs:
            a.record(stream)
            graph.replay()
            b.record(stream)
    stream.synchronize()
    dist = sorted(a.elapsed_time(b) / spg for a, b in evs)
    step_dist = {"n": len(dist), "unit": "ms per step", "median": round(float(np.median(dist)), 5),
                 "p10": round(float(np.percentile(dist, 10)), 5), "p90": round(float(np.percentile(dist, 90)), 5),
                 "how": f"100 replays of the {spg}-step graph, each between its own CUDA events, divided by {spg}"}

    # ---------------- per-kernel durations of the grouped GEMM (same launches) ----------------
    # Each GEMM call (its preparation pass included) replayed from a CUDA graph, alternating the
    # two weight copies, between CUDA events on the launch stream: the launch conditions of the
    # graph-replayed step, without its other kernels.
    lay = layers[0]
    with torch.cuda.stream(stream):
        rt = api.moe_route_permute(logits, k)
        if not fused:
            api.moe_route_permute(logits, k, out=lay.rt, ws=lay.route_ws)
    stream.synchronize()
    n_k = 20

    def gemm_graph(which):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n_k):
                gu_c, gu_s, dn_c, dn_s = layers[i % copies].w
                if which == "gu":
                    api.moe_w4a16_gmm(x, lay.rt.sorted_pair, k, gu_c, gu_s, lay.rt.expert_offsets, T * k,
                                      api.W4_EPI_GELU_GATE, out=lay.h)
                else:
                    api.moe_w4a16_gmm(lay.h, None, 1, dn_c, dn_s, lay.rt.expert_offsets, T * k,
                                      api.W4_EPI_NONE, out=lay.o)
        return g

    t_k = {}
    for which in (() if fused else ("gu", "dn")):
        g = gemm_graph(which)
        with torch.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        stream.synchronize()
        t_k[which] = e0.elapsed_time(e1) / 1e3 / (reps * n_k)
        del g
    t_gu, t_dn = t_k.get("gu", 0.0), t_k.get("dn", 0.0)
    counts = np.diff(rt.expert_offsets.cpu().numpy())
    b_gu, b_dn, hit = gmm_bytes(counts, T, k, H, I)
    hbm_peak, tc_peak, tc_sus, peak_src = peaks()
    prefill = args.workload == "moe_prefill"
    # kernels per step: decode = route, (preparation pass + GEMM) x 2, combine; prefill = two-launch
    # route, (conversion + weight-row exponents + GEMM) x 2, combine
    kernels = 9 if prefill else (1 if fused else 6)
    if fused:
        # one launch per step: the fused kernel's roofline is the step's algorithmic bytes over the
        # step time (its routing, preparation and combine phases included)
        t_step = ms_per_step / 1e3
        achieved = (b_gu + b_dn) / t_step / 1e9
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                    "frac": round(achieved / hbm_peak, 4),
                    "traffic": read_profile_traffic("fused_layer_moe_decode.md", "fused.cu"),
                    "kernel": "moe_layer_kernel (the whole step: one cooperative launch, graph-replayed)",
                    "algorithmic_bytes_per_step": int(b_gu + b_dn), "experts_hit": hit,
                    "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"}
    elif prefill:
        # many routed rows per expert: the tensor-memory kernel, a tensor-core roofline on the
        # GEMMs' algorithmic FLOPs (each launch timed alone: the burst peak)
        flops = 2.0 * T * k * (2 * I * H + H * I)
        roofline = {"bound": "tensor", "achieved": round(flops / (t_gu + t_dn) / 1e12, 1), "peak": tc_peak,
                    "unit": "TFLOP/s", "frac": round(flops / (t_gu + t_dn) / 1e12 / tc_peak, 4),
                    "traffic": read_profile_traffic("tm_gemm_moe_prefill.md", "tm_gemm.cu"),
                    "kernel": "tm_gemm_kernel with its fp16 conversion pass (gate/up + down calls of one step, graph-replayed)",
                    "algorithmic_flops_per_step": flops,
                    "us_gate_up": round(t_gu * 1e6, 2), "us_down": round(t_dn * 1e6, 2),
                    "peak_source": f"{peak_src} (MEASURED_PEAKS.json bf16_tflops, burst)"}
    else:
        achieved = (b_gu + b_dn) / (t_gu + t_dn) / 1e9
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                    "frac": round(achieved / hbm_peak, 4),
                    "traffic": read_profile_traffic(f"stream_gemm_{args.workload}.md"),
                    "kernel": "stream_gemm_kernel with its preparation pass (gate/up + down calls of one step, graph-replayed)",
                    "algorithmic_bytes_per_step": int(b_gu + b_dn), "experts_hit": hit,
                    "us_gate_up": round(t_gu * 1e6, 2), "us_down": round(t_dn * 1e6, 2),
                    "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"}

    # ---------------- end to end through the public API with host buffers ----------------
    # Each step: the pinned host x and logits copied in, the layer's public calls, y copied back
    # to pinned host memory.  A step is captured once into a CUDA graph (copies included); two
    # such graphs, each with its own device buffers and layer, alternate on two streams, so the
    # copies of one step overlap the kernels of the other, as a serving loop pipelines them.
    x_h = torch.empty_like(x, device="cpu").pin_memory()
    x_h.copy_(x.cpu())
    lg_h = torch.empty_like(logits, device="cpu").pin_memory()
    lg_h.copy_(logits.cpu())
    e2e_streams = [torch.cuda.Stream(device), torch.cuda.Stream(device)]
    e2e_bufs = []
    for b in range(2):
        xd, ld = torch.empty_like(x), torch.empty_like(logits)
        yh = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()
        st = e2e_streams[b]
        with torch.cuda.stream(st):
            for _ in range(3):                       # warm-up (and workspace sizing) on this stream
                xd.copy_(x_h, non_blocking=True)
                ld.copy_(lg_h, non_blocking=True)
                yh.copy_(layers[b](xd, ld), non_blocking=True)
        st.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            xd.copy_(x_h, non_blocking=True)
            ld.copy_(lg_h, non_blocking=True)
            yh.copy_(layers[b](xd, ld), non_blocking=True)
        e2e_bufs.append((g, xd, ld, yh))
    torch.cuda.synchronize()
    n_e2e = min(args.steps, 1000) // 2 * 2
    for b in range(2):                               # one replay each before timing
        with torch.cuda.stream(e2e_streams[b]):
            e2e_bufs[b][0].replay()
    torch.cuda.synchronize()
    ranks_barrier(world)
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    e_side = torch.cuda.Event()
    s0, s1 = e2e_streams
    f0.record(s0)
    s1.wait_event(f0)
    for i in range(n_e2e):
        with torch.cuda.stream(e2e_streams[i % 2]):
            e2e_bufs[i % 2][0].replay()
    e_side.record(s1)
    s0.wait_event(e_side)
    f1.record(s0)
    torch.cuda.synchronize()
    ms_e2e = ranks_max(f0.elapsed_time(f1), world, device)
    e2e_value = job_throughput(T * n_e2e, world, ms_e2e)
    del e2e_bufs

    secondary = {}
    if not args.no_secondary and rank == 0:
        secondary = run_secondary(args, device, stream)

    cpu_base = None
    parity = None
    if rank == 0 and world == 1:
        with torch.cuda.stream(stream):
            y_dev = layers[0](x, logits).float().cpu().numpy()
        stream.synchronize()
        ref = {}
        cpu_base = cpu_baseline(case, ref)
        parity = parity_stats(y_dev, ref, rt)

    del graph                    # (holds no collective) released before the group goes
    ranks_finish(world)
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded: codes uniform over -8..7, scales 0.01|N(0,1)|+1e-4, x and logits N(0,1))",
        "config": {"workload": wl["name"], "tokens_per_step": T, "experts": E, "top_k": k,
                   "hidden": H, "intermediate": I, "group": 32, "parallelism": f"replicas{world}",
                   "l2": f"no flush: {copies} weight copies of 428 MB alternate, each step streams the "
                         f"{hit} experts hit (>126 MB L2)",
                   "path": args.path,
                   "timing": f"CUDA graphs of {spg} consecutive steps ({'1 fused call' if fused else '4 calls'}, "
                             f"{kernels} kernel(s) each; weight copies alternating), replayed {args.steps // spg} "
                             f"times; CUDA events on the launch stream"},
        "clocks": clocks.summary(),
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT,
                "h2d_bytes_per_step": int(x.numel() * 2 + logits.numel() * 4),
                "d2h_bytes_per_step": int(T * H * 2),
                "how": f"public API (MoELayer) per step: pinned H2D of x and logits, "
                       f"{'1 fused call' if fused else '4 calls'} ({kernels} kernel(s)), D2H of y to pinned "
                       f"host memory, captured per step in a CUDA graph; two graphs with their own buffers "
                       f"alternate on two streams ({n_e2e} steps), so one step's copies overlap the other's "
                       f"kernels"},
        "gpu_launches": kernels * args.steps,
        "step_time_distribution": step_dist,
        "roofline": roofline,
        "cpu_baseline": cpu_base,
        "parity": parity,
        "secondary": secondary,
    }
    print(json.dumps(line), flush=True)


def _physical_gpu_index(local):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        items = [v.strip() for v in vis.split(",") if v.strip()]
        if local < len(items) and items[local].isdigit():
            return int(items[local])
    return local


def cpu_baseline(case, outputs=None):
    """The oracle as it stands on a bounded sample of the same workload (host cores).  When
    `outputs` is a dict, it receives the sampled tokens, their oracle outputs and the routing."""
    import numpy as np

    from oracle import moe
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=os.cpu_count())
    except Exception:
        threads = os.cpu_count()
    # chunks of 8 tokens until about 10 s of host work (at most every token of the layer)
    done, chunk, budget_s = 0, 8, 10.0
    t0 = time.perf_counter()
    ys = []
    while done < case.T and time.perf_counter() - t0 < budget_s:
        tokens = np.arange(done, min(done + chunk, case.T))
        res = moe.moe_layer(case.x, case.logits, case.gu_codes, case.gu_scales, case.dn_codes, case.dn_scales,
                            case.k, tokens=tokens)
        if outputs is not None:
            ys.append(res.y[tokens])
            outputs["routing"] = res.routing
        done += len(tokens)
    dt = time.perf_counter() - t0
    if outputs is not None:
        outputs["tokens"] = np.arange(done)
        outputs["y"] = np.concatenate(ys) if ys else np.zeros((0, case.H))
    # the same oracle on one host thread, on the first chunk only
    one = None
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            t1 = time.perf_counter()
            moe.moe_layer(case.x, case.logits, case.gu_codes, case.gu_scales, case.dn_codes, case.dn_scales,
                          case.k, tokens=np.arange(0, min(chunk, case.T)))
            one = min(chunk, case.T) / (time.perf_counter() - t1)
    except Exception:
        pass
    return {"value": round(done / dt, 3), "unit": UNIT, "cores": int(threads), "kind": "oracle",
            "value_1_thread": None if one is None else round(one, 3),
            "sample": f"{done} of {case.T} tokens of the same layer in chunks of {chunk} (routing of "
                      f"all {case.T} each chunk); {dt:.1f} s of float64 numpy on the host; "
                      f"value_1_thread: the first chunk with the BLAS pool limited to one thread"}


def parity_stats(y_dev, ref, rt_dev=None):
    """Parity of the device's layer output with the oracle's on the cpu_baseline sample: per token
    row rel-L2 and max-abs error (as a fraction of the row's max |ref|) against the tolerance, and
    the routing compared bit for bit over every token."""
    import numpy as np
    tok = ref["tokens"]
    if tok.size == 0:
        return None
    y = np.asarray(y_dev, dtype=np.float64)[tok]
    r = np.asarray(ref["y"], dtype=np.float64)
    nref = np.linalg.norm(r, axis=1)
    rel = np.linalg.norm(y - r, axis=1) / np.where(nref > 0, nref, 1.0)
    mref = np.abs(r).max(axis=1)
    mabs = np.abs(y - r).max(axis=1) / np.where(mref > 0, mref, 1.0)
    ok = (rel <= 5e-3) & (mabs <= 2e-2)
    out = {"tokens_checked": int(tok.size), "max_rel_l2": float(f"{rel.max():.3e}"),
           "median_rel_l2": float(f"{np.median(rel):.3e}"), "max_abs_frac": float(f"{mabs.max():.3e}"),
           "rows_within_tolerance": int(ok.sum()), "tolerance": {"rel_l2": 5e-3, "max_abs_frac": 2e-2},
           "reference": "the CPU oracle (float64) on the cpu_baseline sample"}
    if rt_dev is not None and "routing" in ref:
        ro = ref["routing"]
        out["routing_bit_exact"] = {
            "topk_ids": bool(np.array_equal(rt_dev.topk_ids.cpu().numpy(), ro.topk_ids)),
            "expert_offsets": bool(np.array_equal(rt_dev.expert_offsets.cpu().numpy(), ro.expert_offsets)),
            "sorted_pair": bool(np.array_equal(rt_dev.sorted_pair.cpu().numpy(), ro.sorted_pair)),
            "pair_pos": bool(np.array_equal(rt_dev.pair_pos.cpu().numpy(), ro.pair_pos))}
    return out


def run_secondary(args, device, stream):
    """Other configurations of the same kernels, timed briefly (not the headline)."""
    import numpy as np
    import torch

    from w4a16_group_quantized_w4_b200 import api, synth
    out = {}
    hbm_peak, _, _, _ = peaks()
    # the small dense linear (M = 4, K = 256, N = 256; launch-latency bound): graph-replayed calls
    c1 = synth.case_dense_small()
    xx, cc, ss = to_dev(c1.x, "bf16", device), to_dev(c1.codes, "u32", device), to_dev(c1.scales, "bf16", device)
    yy = torch.empty((c1.M, c1.N), dtype=torch.bfloat16, device=device)
    with torch.cuda.stream(stream):
        for _ in range(5):
            api.w4a16_linear(xx, cc, ss, y=yy)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(20):
                api.w4a16_linear(xx, cc, ss, y=yy)
        g.replay()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(10):
            g.replay()
        e1.record(stream)
    stream.synchronize()
    out["dense_small_M4_K256_N256"] = {"us_per_call": round(e0.elapsed_time(e1) * 1e3 / 200, 2),
                                       "how": "200 calls in graphs of 20 (preparation pass + GEMM each)"}
    del g
    # dense decode GEMV, K=4096, N=14336: 8 rotating weight copies (264 MB > 2x L2)
    base = synth.case_dense_gemv(16)
    nc = 8
    codes = [to_dev(base.codes, "u32", device) for _ in range(nc)]
    scales = [to_dev(base.scales, "bf16", device) for _ in range(nc)]
    for M in (1, 4, 16):
        xx = to_dev(base.x[:M], "bf16", device)
        yy = torch.empty((M, 14336), dtype=torch.bfloat16, device=device)
        with torch.cuda.stream(stream):
            for i in range(10):
                api.w4a16_linear(xx, codes[i % nc], scales[i % nc], y=yy)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(nc):
                    api.w4a16_linear(xx, codes[i], scales[i], y=yy)
            g.replay()
        stream.synchronize()
        reps = 50
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        stream.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (reps * nc)
        byts = 14336 * 4096 // 2 + 14336 * 128 * 2 + M * 4096 * 2 + M * 14336 * 2
        out[f"dense_gemv_M{M}_K4096_N14336"] = {"us": round(us, 2), "GB/s": round(byts / us / 1e3, 1),
                                                 "frac_hbm": round(byts / us / 1e3 / hbm_peak, 3)}
        del g
    del codes, scales
    torch.cuda.empty_cache()
    # MoE prefill layer (8192 tokens, Zipf-skewed experts), a few steps
    if args.workload != "moe_prefill":
        pc = synth.case_moe_prefill(args.seed)
        lay = api.MoELayer(to_dev(pc.gu_codes, "u32", device), to_dev(pc.gu_scales, "bf16", device),
                           to_dev(pc.dn_codes, "u32", device), to_dev(pc.dn_scales, "bf16", device),
                           pc.T, pc.k)
        xx, ll = to_dev(pc.x, "bf16", device), to_dev(pc.logits, "f32", device)
        with torch.cuda.stream(stream):
            for _ in range(3):
                lay(xx, ll)
        stream.synchronize()
        reps = 5
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                lay(xx, ll)
            e1.record(stream)
        stream.synchronize()
        ms = e0.elapsed_time(e1) / reps
        flops = 2.0 * pc.T * pc.k * (2 * 704 * 2816 + 2816 * 704)
        _, tc_peak, _, _ = peaks()
        out["moe_prefill_T8192_zipf1.1"] = {"ms": round(ms, 3), "tokens/s": round(pc.T / ms * 1e3, 1),
                                            "TFLOP/s": round(flops / ms / 1e9, 1),
                                            "frac_bf16_peak": round(flops / ms / 1e9 / tc_peak, 3)}
        del lay
        torch.cuda.empty_cache()
    out.update(run_fused(device, stream))
    out.update(run_stack(device, stream, L=args.stack_layers))
    return out


def run_fused(device, stream):
    """The single-launch fused layer (moe_w4a16_layer) against the four-call path on the decode
    configuration at 1, 8 and 64 tokens: graph-replayed steps alternating two weight copies (856
    MB, beyond L2), the same y bit for bit."""
    import numpy as np
    import torch

    from w4a16_group_quantized_w4_b200 import api, synth
    E, k, H, I = 128, 8, 2816, 704
    case = synth.moe_case(64, E, k, H, I, seed=7)
    W = [(to_dev(case.gu_codes, "u32", device), to_dev(case.gu_scales, "bf16", device),
          to_dev(case.dn_codes, "u32", device), to_dev(case.dn_scales, "bf16", device)) for _ in range(2)]
    xs, ls = to_dev(case.x, "bf16", device), to_dev(case.logits, "f32", device)
    res = {}
    for T in (1, 8, 64):
        x, lg = xs[:T].contiguous(), ls[:T].contiguous()
        row = {}
        ys = {}
        for name, fused in (("four_call", False), ("fused", True)):
            lays = [api.MoELayer(*W[c], T, k, fused=fused) for c in range(2)]
            with torch.cuda.stream(stream):
                for i in range(3):
                    lays[i % 2](x, lg)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for i in range(10):
                        lays[i % 2](x, lg)
                g.replay()
            stream.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(30):
                    g.replay()
                e1.record(stream)
            stream.synchronize()
            row[f"{name}_us"] = round(e0.elapsed_time(e1) * 1e3 / 300, 2)
            with torch.cuda.stream(stream):
                ys[name] = lays[1](x, lg).clone()
            stream.synchronize()
            del g, lays
        row["bit_identical"] = bool(torch.equal(ys["fused"].view(torch.int16), ys["four_call"].view(torch.int16)))
        res[f"moe_layer_fused_vs_four_call_T{T}"] = row
    del W
    torch.cuda.empty_cache()
    return res


def run_stack(device, stream, L=30, reps=3):
    """Repack + full expert stack: 30 layers x 128 experts of planted bf16 weights (generated on
    the device), repacked, then decode steps through all 30 chained layers (layer l + 1 takes
    moe_rms_chain of layer l's output) at 1, 32 and 256 tokens."""
    import torch

    from w4a16_group_quantized_w4_b200 import stack, synth, synth_device
    res = {}
    hbm_peak, _, _, _ = peaks()
    st = stack.MoEStack(L)
    H, I, E = st.H, st.I, st.E
    w_gu = synth_device.planted(st.gate_up_rows() * H // 32, 0, 0, 500).view(st.gate_up_rows(), H)
    w_dn = synth_device.planted(st.down_rows() * I // 32, 0, 0, 501).view(st.down_rows(), I)
    with torch.cuda.stream(stream):
        rep = st.repack(w_gu, w_dn, stream=stream)          # warm-up (also the parity-checked result)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            st.repack(w_gu, w_dn, stream=stream)
        e1.record(stream)
    stream.synchronize()
    ms = e0.elapsed_time(e1) / reps
    groups = (st.gate_up_rows() * H + st.down_rows() * I) // 32
    moved = groups * (64 + 16 + 2 + 1)          # bf16 in; codes, scale, group_m out
    res[f"repack_{L}x128_experts"] = {"ms": round(ms, 3), "groups": groups, "GB/s": round(moved / ms / 1e6, 1),
                                    "frac_hbm": round(moved / ms / 1e6 / hbm_peak, 3),
                                    "off_grid": rep.off_grid_gate_up + rep.off_grid_down}
    del w_gu, w_dn, rep
    torch.cuda.empty_cache()
    for T in (1, 32, 256):
        x0 = to_dev(synth.bf16_normal((T, H), 0, 600), "bf16", device)
        lgs = [to_dev(synth.router_logits(T, E, 0, 700 + l), "f32", device) for l in range(L)]
        for fused in (False, True):
            if fused and not st.fusable(T):
                continue
            with torch.cuda.stream(stream):
                for _ in range(2):
                    st.chained_step(x0, lgs, stream=stream, fused=fused)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    st.chained_step(x0, lgs, stream=stream, fused=fused)
                g.replay()
            stream.synchronize()
            hit = sum(int((torch.diff(st.layer(l, T).rt.expert_offsets) > 0).sum()) for l in range(L))
            n = 20
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(n):
                    g.replay()
                e1.record(stream)
            stream.synchronize()
            ms = e0.elapsed_time(e1) / n
            byts = hit * st.expert_bytes() + L * T * H * 2 * 2 + (L - 1) * T * H * 2 * 2   # + the chaining
            res[f"stack_decode_{L}_layers_T{T}" + ("_fused" if fused else "")] = {
                "ms_per_step": round(ms, 3), "tokens/s": round(T / ms * 1e3, 1), "experts_hit": hit,
                "GB/s": round(byts / ms / 1e6, 1), "frac_hbm": round(byts / ms / 1e6 / hbm_peak, 3)}
            del g
    del st
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------------------------------
# reference arm: the CPU oracle on the same workload
# ------------------------------------------------------------------------------------------

def reference(args, world, rank):
    if rank != 0:
        return
    import numpy as np

    from oracle import moe
    from w4a16_group_quantized_w4_b200 import synth
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=os.cpu_count())
    except Exception:
        threads = os.cpu_count()
    wl = WORKLOADS[args.workload]
    if args.workload == "dense_gemv":
        print(json.dumps({"impl": "reference", "unavailable": "the reference arm times the MoE workloads only"}),
              flush=True)
        return
    case = synth.moe_case(wl["T"], 128, 8, 2816, 704, seed=args.seed, zipf_s=wl["zipf"])
    budget_s = 150.0

    def step(i):
        t = i % case.T
        moe.moe_layer(case.x, case.logits, case.gu_codes, case.gu_scales, case.dn_codes,
                      case.dn_scales, case.k, tokens=[t])

    t0 = time.perf_counter()
    step(0)
    one = time.perf_counter() - t0
    n_w = min(args.warmup, max(0, int(0.1 * budget_s / one)))
    for i in range(n_w):
        step(i)
    n_run = max(1, min(args.steps, int(0.9 * budget_s / one)))
    t0 = time.perf_counter()
    for i in range(n_run):
        step(i)
    dt = time.perf_counter() - t0
    value = n_run / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": n_run, "steps_requested": args.steps, "warmup": n_w, "ms_per_step": round(dt / n_run * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same seeded inputs as the native arm)",
        "config": {"workload": wl["name"], "tokens_per_step": 1, "experts": 128, "top_k": 8,
                   "hidden": 2816, "intermediate": 704, "group": 32, "parallelism": "host"},
        "cpu_baseline": {"kind": "oracle", "cores": int(threads), "value": round(value, 4), "unit": UNIT,
                         "sample": f"one token of the {case.T}-token layer per step (its 8 expert pairs), "
                                   f"steps capped to a {budget_s:.0f} s budget"},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup(args.gpus)
    if args.impl == "reference":
        reference(args, world, rank)
        return
    native(args, world, rank, local)


if __name__ == "__main__":
    main()
