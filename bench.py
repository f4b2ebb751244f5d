#!/usr/bin/env python
"""Benchmark of the BASA forward hot path (one layer = pool [+ route] + attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload flux2k] [--impl ours|reference]

A step is one layer call over one batch of synthetic inputs already resident in
HBM; consecutive steps walk the workload's shift cycle (one shift per layer).
Rank 0 prints ONE JSON line. Multi-GPU runs (torchrun) time on the device and
report the max over ranks; by default every rank runs its own full copy of the
workload ("scaling": "weak"); with `--shard heads` one layer's (batch, head)
units are split over the ranks ("scaling": "strong"). Either way there is no
exchange on the data path: pooling, routing and attention have no term across heads.

L2: workloads whose inputs exceed the 126 MB L2 are timed back to back; for
smaller ones the line adds `l2_flushed`, every step timed after a 256 MB scratch
write outside the events.

The line also carries: `roofline` (the attention kernel's achieved TFLOP/s from
CUDA events around its launches, against the measured bf16 peak, and its DRAM
traffic from the committed ncu summary when that was taken on the current
source), `hbm_kernels` (the pooling / routing pre-pass against measured HBM
bandwidth), `e2e` (the same metric through BasaLayer.forward with pinned host
buffers, copies of successive steps pipelined over three streams), `clocks`,
`cpu_baseline` and context lines for the other workloads and forms (Wan 480p and
video, the branch form, the text-query rows, the bfloat16 tensor-core backward on
the FLUX 2048^2 and Wan shapes, the float32 backward).

The reference arm (--impl reference) times the float64 CPU oracle on the host
cores on a bounded sample of the same workload (the oracle is the only other
implementation there is).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_window_attention_b200 import accounting, sharding, synth  # noqa: E402

METRIC = "shifted-window attn fwd effective TFLOP/s & % of B200 BF16 peak; ms/layer"
ATTN_SOURCE = os.path.join(ROOT, "sparse_window_attention_b200", "csrc", "attn_bf16_sm100.cu")
L2_BYTES = 126e6
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


def kernel_traffic(kernel_file: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel source (sha256 recorded in the summary); else None."""
    prof = os.path.join(ROOT, "profiles", f"attn_bf16_{workload}.md")
    if not os.path.exists(prof):
        return None
    text = open(prof).read()
    sha = hashlib.sha256(open(kernel_file, "rb").read()).hexdigest()
    m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    m_tr = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_sha or not m_tr or m_sha.group(1) != sha:
        return None
    return float(m_tr.group(1))


_NVML_POLL = r"""
import sys, time
import pynvml
pynvml.nvmlInit()
bus = sys.argv[1]
h = pynvml.nvmlDeviceGetHandleByPciBusId(bus) if bus else pynvml.nvmlDeviceGetHandleByIndex(int(sys.argv[2]))
print("max", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
while True:
    ta = time.time()
    mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
    bits = int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))
    print(f"{ta:.6f} {time.time():.6f} {mhz} {bits}", flush=True)
    time.sleep(0.0005)
"""


class ClockSampler:
    """SM clocks and throttle reasons sampled DURING the timed region.

    A separate process polls NVML every ~0.5 ms (no GIL contention with the
    launching thread) and timestamps each sample; the samples inside the timed
    region's wall-clock interval are kept, so a region of a few ms still gets a
    handful. Without NVML, `nvidia-smi -lms 100` is the fallback."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))
    FIELDS = "clocks.sm,clocks.max.sm,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap"

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.max_mhz = None
        self.source = None
        self.t0 = self.t1 = None

    def __enter__(self):
        bus = ""
        try:
            pr = torch.cuda.get_device_properties(self.index)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen([sys.executable, "-c", _NVML_POLL, bus, str(self.index)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            first = self.proc.stdout.readline().split()
            if len(first) != 2 or first[0] != "max":
                raise OSError("nvml poller did not start")
            self.max_mhz = float(first[1])
            self.source = "nvml from a separate process, every 0.5 ms"
        except Exception:
            if self.proc is not None:
                self.proc.kill()
            self.source = "nvidia-smi -lms 100"
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100", "-i",
                     str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except (FileNotFoundError, OSError):
                self.proc = None
                self.source = None
        if self.proc is not None:
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            # let the poll loop reach its steady rate before the timed region starts
            deadline = time.time() + 2.0
            while len(self.lines) < 2 and time.time() < deadline:
                time.sleep(0.001)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.002)  # let the poller report past the end of the region
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)

    def summary(self):
        sm, mx, reasons = [], self.max_mhz, set()
        nvml = self.source is not None and self.source.startswith("nvml")
        for line in self.lines:
            if nvml:
                # "t mhz bits", or "ta tb mhz bits": a query made over [ta, tb]; kept
                # when it overlaps the timed region
                parts = line.split()
                if len(parts) not in (3, 4):
                    continue
                ta, tb = float(parts[0]), float(parts[-3])
                mhz, bits = float(parts[-2]), int(parts[-1])
                if self.t0 is not None and (tb < self.t0 or ta > self.t1):
                    continue
                sm.append(mhz)
                reasons.update(n for n, b in self.REASONS if bits & b)
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for (n, _), v in zip(self.REASONS, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": self.source}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    return x if world == 1 else sharding.max_over_ranks(x)


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ----------------------------------------------------------------- our arm


def run_ours(args, world, rank, local):
    from sparse_window_attention_b200.layer import BasaLayer

    wl = synth.WORKLOADS[args.workload]
    cnt = accounting.workload_counts(wl)
    shifts = synth.SHIFT_CYCLES[args.workload]
    strong = getattr(args, "shard", "replicas") == "heads"
    if strong:
        # one layer split over the ranks by (batch, head) units: every rank draws the
        # same full inputs and keeps its own units (no exchange on the data path)
        layer = BasaLayer.for_shard(wl.B, wl.heads, wl.d, wl.grid, wl.window, world, rank, pool=wl.pool,
                                    n_text=wl.n_text, routed_k=wl.routed_k, dtype=wl.dtype,
                                    route_radius=wl.route_radius)
        q, k, v = (layer.shard_of(x).contiguous() for x in synth.make_inputs(wl, seed=args.seed))
        unit_frac = (layer.units[1] - layer.units[0]) / (wl.B * wl.heads)
    else:
        q, k, v = synth.make_inputs(wl, seed=args.seed + rank)
        layer = BasaLayer(wl.B, wl.heads, wl.d, wl.grid, wl.window, wl.pool, wl.n_text, wl.routed_k, wl.dtype,
                          route_radius=wl.route_radius)
        unit_frac = 1.0
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out = torch.empty_like(qd)
    stream = torch.cuda.current_stream()

    fused = layer.fused and all(layer.fused_bytes(sh) > 0 for sh in shifts)

    def step(i, ev=None):
        sh = shifts[i % len(shifts)]
        if ev is not None:
            ev[0].record(stream)
        if fused:  # pooled K/V and routing in one pass over q, k, v
            layer.pool_route(qd, kd, vd, sh)
        elif layer.has_pool:
            layer.pool_kv(kd, vd, sh)
        if ev is not None:
            ev[1].record(stream)
        if layer.routed_k > 0 and not fused:
            layer.route(qd, kd, sh)
        if ev is not None:
            ev[2].record(stream)
        layer.attention(qd, kd, vd, out, sh)
        if ev is not None:
            ev[3].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    assert layer.device_error() == 0

    # timed region: K whole steps
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    with sampler:
        sampler.mark_start()
        t0.record(stream)
        for i in range(args.steps):
            step(i)
        t1.record(stream)
        torch.cuda.synchronize()
        sampler.mark_end()
    barrier(world)
    step_ms = t0.elapsed_time(t1) / args.steps
    step_ms = max_over_ranks(step_ms, world)
    assert layer.device_error() == 0

    # attention-kernel duration (events bracketing each attention launch)
    n_ev = min(args.steps, 200)
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(n_ev)]
    for i in range(n_ev):
        step(i, evs[i])
    torch.cuda.synchronize()
    l2_flushed = None
    if cnt["attn_bytes"] < L2_BYTES:
        # the inputs fit in L2: also time every step after a 256 MB scratch write
        # (outside the events), which evicts them, so the kernels read from HBM
        scratch = torch.empty(256 << 20, dtype=torch.uint8, device=qd.device)
        fevs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(n_ev)]
        for i in range(n_ev):
            scratch.fill_(i & 0xFF)
            step(i, fevs[i])
        torch.cuda.synchronize()
        del scratch
        f_step = statistics.mean(e[0].elapsed_time(e[3]) for e in fevs)
        f_attn = statistics.mean(e[2].elapsed_time(e[3]) for e in fevs)
        f_pool = statistics.mean(e[0].elapsed_time(e[1]) for e in fevs)
        f_route = statistics.mean(e[1].elapsed_time(e[2]) for e in fevs)
        f_ach = cnt["attn_flops"] / (f_attn * 1e-3) / 1e12
        peaks0, _ = load_peaks()
        l2_flushed = {
            "how": "256 MB scratch write before every step, outside the CUDA events; step = pool start to attention end",
            "steps": n_ev,
            "ms_per_step": round(f_step, 4),
            "value": round(cnt["attn_flops"] / (f_step * 1e-3) / 1e12, 2),
            "attn_ms": round(f_attn, 4),
            "attn_frac_of_measured_bf16": round(f_ach / peaks0["bf16_tflops"], 4),
            "hbm_kernels": hbm_lines(cnt, f_pool, f_route, peaks0["hbm_gbs"], fused),
        }
    attn_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    pool_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    route_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    # the attention kernel at each shift of the cycle alone (window types differ per shift)
    per_shift = {}
    for i, e in enumerate(evs):
        per_shift.setdefault(str(tuple(shifts[i % len(shifts)])), []).append(e[2].elapsed_time(e[3]))
    per_shift_ms = {k: round(statistics.mean(v), 4) for k, v in per_shift.items()}

    flops = cnt["attn_flops"]
    # whole-job throughput: the full layer split over the ranks (strong) or one
    # full layer per rank (weak); the per-rank kernel does unit_frac of a layer
    value = (1 if strong else world) * flops / (step_ms * 1e-3) / 1e12
    peaks, peak_kind = load_peaks()
    peak = peaks["bf16_tflops"]
    achieved = unit_frac * flops / (attn_ms * 1e-3) / 1e12
    traffic = kernel_traffic(ATTN_SOURCE, args.workload)
    clocks = sampler.summary()
    res = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": True,
        "scaling": "strong" if strong else "weak",
        "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": workload_config(wl, world, strong),
        "dense_equivalent": {
            "note": "context only: the dense attention this layer replaces, at the measured step time",
            "sparsity": round(accounting.sparsity(cnt["keys_per_query"], wl.N + wl.n_text), 4),
            "tflops": round(world * accounting.dense_attn_flops(wl.B, wl.heads, wl.N, wl.d, wl.N + wl.n_text)
                            / (step_ms * 1e-3) / 1e12, 1),
        },
        "pct_of_peak": {
            "step_vs_measured_burst": round(value / world / peak, 4),
            "step_vs_nominal_2250": round(value / world / 2250.0, 4),
            "attn_kernel_vs_nominal_2250": round(achieved / 2250.0, 4),
        },
        "roofline": {
            "kernel": "attn_bf16_kernel",
            "bound": "tensor",
            "achieved": round(achieved, 2),
            "peak": peak,
            "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "peak_source": f"{peak_kind} bf16 burst (MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback 1.59 PF/s",
            "traffic": traffic,
            "attn_ms": round(attn_ms, 4),
            "attn_ms_per_shift": per_shift_ms,
        },
        "hbm_kernels": hbm_lines(cnt, pool_ms, route_ms, peaks["hbm_gbs"], fused),
        "clocks": clocks,
        "l2_flushed": l2_flushed,
        "gpu_launches": args.steps * layer.launches_per_forward(),
    }
    if not args.no_e2e:
        res["e2e"] = run_e2e(args, layer, q, k, v, shifts, flops, world, 1 if strong else world)
    if not args.no_extra and world == 1:
        res["branch_form"] = run_branch_form(args, layer, qd, kd, vd, shifts, flops)
        if wl.n_text > 0:
            res["text_queries"] = run_text_queries(args, layer, wl, kd, vd)
        res["backward_bf16"] = {n: run_backward_bf16(args, n, synth.SHIFT_CYCLES[n][-1]) for n in ("flux2k", "wan")}
        res["backward_f32"] = run_backward(args)
        for name in ("wan", "wan_video", "flux1k", "flux4k"):
            if args.workload != name:
                res["also_" + name] = run_also(args, name)
    return res


def run_text_queries(args, layer, wl, kd, vd):
    """The text-query rows of the joint layer: dense attention of the n_text text
    queries over all N + n_text keys (4 d FLOPs per query-key pair)."""
    g = torch.Generator(device="cpu").manual_seed(args.seed + 100)
    qt = torch.randn(wl.B, wl.heads, wl.n_text, wl.d, generator=g).to(kd.dtype).cuda()
    out = torch.empty_like(qt)
    steps = max(20, args.steps // 4)
    for _ in range(3):
        layer.text_attention(qt, kd, vd, out)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        layer.text_attention(qt, kd, vd, out)
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    flops = 4.0 * wl.d * wl.B * wl.heads * wl.n_text * (wl.N + wl.n_text)
    peaks, _ = load_peaks()
    achieved = flops / (ms * 1e-3) / 1e12
    return {"ms": round(ms, 4), "gflop": round(flops / 1e9, 2), "value": round(achieved, 2), "unit": "TFLOP/s",
            "frac_of_measured_bf16": round(achieved / peaks["bf16_tflops"], 4),
            "workspace_bytes": layer.text_workspace.numel() if layer.text_workspace is not None else 0}


def run_backward(args):
    """Context: the float32 backward (CUDA cores) on the FLUX 1024^2 shape in float32,
    counted as 10 d FLOPs per query-key pair (S recomputed, dP, dQ, dK, dV)."""
    import dataclasses

    from sparse_window_attention_b200 import binding as B
    from sparse_window_attention_b200.layer import BasaLayer

    wl = dataclasses.replace(synth.WORKLOADS["flux1k"], dtype="f32", name="flux1k_f32")
    sh = (0, 8, 8)
    q, k, v = synth.make_inputs(wl, seed=args.seed)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    layer = BasaLayer(wl.B, wl.heads, wl.d, wl.grid, wl.window, wl.pool, wl.n_text, wl.routed_k, wl.dtype)
    layer.pool_kv(kd, vd, sh)
    out = torch.empty_like(qd)
    lse = torch.empty(qd.shape[:-1], dtype=torch.float32, device=qd.device)
    layer.attention_lse(qd, kd, vd, out, lse, sh, B.BASA_KEYS_ALL)
    dout = torch.randn_like(qd)
    for _ in range(2):
        layer.backward(qd, kd, vd, out, lse, dout, sh)
    torch.cuda.synchronize()
    steps = 5
    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        layer.backward(qd, kd, vd, out, lse, dout, sh)
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    cnt = accounting.workload_counts(wl)
    flops = 2.5 * cnt["attn_flops"]
    return {"workload": "flux1k shape, float32, shift (0, 8, 8)", "ms": round(ms, 3),
            "gflop": round(flops / 1e9, 2), "value": round(flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "note": "CUDA-core float32 with atomic dK/dV accumulation (the bfloat16 backward runs on the tensor cores: "
                    "backward_bf16)"}


def run_backward_bf16(args, name, shift):
    """The tensor-core backward (bfloat16) of one layer of workload `name` at `shift`:
    dq, dk, dv from the forward's output and log-sum-exp. Algorithmic FLOPs = 2.5 x
    the forward's (the five products S, dP, dq, dK, dV); the kernels execute 3.5 x
    (the dK/dV pass recomputes S and dP instead of accumulating dq with atomics)."""
    from sparse_window_attention_b200 import binding as B
    from sparse_window_attention_b200.layer import BasaLayer

    wl = synth.WORKLOADS[name]
    q, k, v = synth.make_inputs(wl, seed=args.seed)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    layer = BasaLayer(wl.B, wl.heads, wl.d, wl.grid, wl.window, wl.pool, wl.n_text, wl.routed_k, wl.dtype,
                      route_radius=wl.route_radius)
    layer.forward(qd, kd, vd, shift)  # pooled K/V and routes
    out = torch.empty_like(qd)
    lse = torch.empty(qd.shape[:-1], dtype=torch.float32, device=qd.device)
    layer.attention_lse(qd, kd, vd, out, lse, shift, B.BASA_KEYS_ALL)
    g = torch.Generator(device="cpu").manual_seed(args.seed + 7)
    dout = torch.randn(qd.shape, generator=g).to(torch.bfloat16).cuda()
    for _ in range(3):
        layer.backward(qd, kd, vd, out, lse, dout, shift)
    torch.cuda.synchronize()
    steps = max(10, args.steps // 10)
    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        layer.backward(qd, kd, vd, out, lse, dout, shift)
    t1.record(stream)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    ms = t0.elapsed_time(t1) / steps
    cnt = accounting.workload_counts(wl)
    alg = 2.5 * cnt["attn_flops"]
    executed = 3.5 * cnt["attn_flops"]
    peaks, _ = load_peaks()
    return {"workload": f"{name}, shift {tuple(shift)}, bfloat16", "ms": round(ms, 4),
            "algorithmic_gflop": round(alg / 1e9, 2), "value": round(alg / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "frac_of_measured_bf16": round(alg / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
            "executed_tensor_tflops": round(executed / (ms * 1e-3) / 1e12, 2),
            "executed_frac_of_measured_bf16": round(executed / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
            "launches_per_step": 5 if (layer.has_pool or layer.n_text) else 3,
            "note": "records + dq pass + pooled/text dK/dV chunks + chunk reduction + window dK/dV; deterministic"}


def run_branch_form(args, layer, qd, kd, vd, shifts, flops):
    """The same layer in the branch form (BASA §A.1): local windows and the pooled +
    text keys as two attention calls with log-sum-exp, then their merge. Context
    for the single-pass kernel, which needs neither the second pass over Q nor the
    merge."""
    from sparse_window_attention_b200 import binding as B

    groups = (B.BASA_KEYS_POOLED if layer.has_pool else 0) | (B.BASA_KEYS_TEXT if layer.n_text else 0)
    if not groups:
        return None
    splits = [B.BASA_KEYS_WINDOWS, groups]
    out = torch.empty_like(qd)
    steps = max(10, args.steps // 10)
    for i in range(3):
        layer.forward_branches(qd, kd, vd, shifts[i % len(shifts)], splits, out=out)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        layer.forward_branches(qd, kd, vd, shifts[i % len(shifts)], splits, out=out)
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    return {"splits": "windows | pooled + text", "ms_per_step": round(ms, 4),
            "value": round(flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "launches_per_step": layer.launches_per_forward() + len(splits)}


def workload_config(wl, world, strong=False):
    """The `config` object of the JSON line (the same for both arms)."""
    cnt = accounting.workload_counts(wl)
    shifts = synth.SHIFT_CYCLES[wl.name]
    return {
        "workload": f"{wl.name}: B={wl.B} heads={wl.heads} d={wl.d} grid={'x'.join(map(str, wl.grid))} "
                    f"window={'x'.join(map(str, wl.window))} shifts={shifts} pool={'x'.join(map(str, wl.pool))} "
                    f"text={wl.n_text} routed_k={wl.routed_k}"
                    + (f" route_radius={wl.route_radius}" if wl.route_radius else ""),
        "keys_per_query": cnt["keys_per_query"],
        "attn_gflop_per_layer": round(cnt["attn_flops"] / 1e9, 2),
        "parallelism": (f"one layer's {wl.B * wl.heads} (batch, head) units split over {world} GPU(s) "
                        "(sharding.unit_shard), no data-path collective" if strong else
                        f"replicas: a full layer ({wl.B * wl.heads} (batch, head) units) per GPU on each of "
                        f"{world} GPU(s), no data-path collective"),
        "l2": (f"inputs {cnt['attn_bytes'] / 1e6:.0f} MB > 126 MB L2; no flush" if cnt["attn_bytes"] >= L2_BYTES else
               f"inputs {cnt['attn_bytes'] / 1e6:.0f} MB < 126 MB L2: the headline times back-to-back steps (warm "
               "L2); `l2_flushed` times every step after a 256 MB scratch write"),
    }


def hbm_lines(cnt, pool_ms, route_ms, hbm_gbs, fused):
    """Achieved bandwidth of the HBM-bound pre-pass: compulsory bytes / event time."""
    def line(ms, nbytes, what):
        if not nbytes:
            return None
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"ms": round(ms, 4), "bytes": nbytes, "GB/s": round(gbs, 1), "frac_of_measured_hbm": round(gbs / hbm_gbs, 4),
                "launches": what}

    if fused:
        # one read of q, k, v + pooled K/V written; partial sums and top-k are inside the time
        return {"pool_route_fused": line(pool_ms, cnt["pool_route_bytes"],
                                         "pool + window partial sums, partial reduction, top-k")}
    return {"pool_kv": line(pool_ms, cnt["pool_bytes"], "box means over pool patches"),
            "route": line(route_ms, cnt["route_bytes"], "box means over windows, top-k")}


def run_e2e(args, layer, q, k, v, shifts, flops, world, job_layers=None):
    """Same metric through the public API with host (pinned) buffers: every step
    copies its q, k, v host->device, runs the layer and copies the output back.
    Steps are pipelined over three streams with two device buffer sets: the inputs
    of step i + 1 travel host->device while step i computes and step i - 1's output
    travels device->host (PCIe is full duplex); every step's copies are inside the
    timed region, which runs from the first input copy to the last output copy."""
    job_layers = world if job_layers is None else job_layers  # full layers the job computes per step
    hq, hk, hv = q.pin_memory(), k.pin_memory(), v.pin_memory()
    hout = torch.empty_like(hq).pin_memory()
    sets = [tuple(torch.empty_like(x, device="cuda") for x in (hq, hk, hv)) for _ in range(2)]
    outs = [torch.empty_like(sets[0][0]) for _ in range(2)]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    steps = max(3, min(args.steps, args.e2e_steps))

    def step(i):
        b = i % 2
        dq, dk, dv = sets[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[b])  # step i - 2 no longer reads this set
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            in_done[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_done[b])
            if i >= 2:
                s_comp.wait_event(out_done[b])  # step i - 2's output has left this buffer
            layer.forward(dq, dk, dv, shifts[i % len(shifts)], out=outs[b], stream=s_comp)
            comp_done[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            hout.copy_(outs[b], non_blocking=True)
            out_done[b].record(s_out)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(steps):
        step(i)
    t1.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world)
    esz = hq.element_size()
    return {
        "value": round(job_layers * flops / (ms * 1e-3) / 1e12, 2),
        "unit": "TFLOP/s",
        "ms_per_step": round(ms, 3),
        "steps": steps,
        "h2d_bytes_per_step": (hq.numel() + hk.numel() + hv.numel()) * esz,
        "d2h_bytes_per_step": hout.numel() * esz,
        "pipelining": "3 streams (copy in / compute / copy out), 2 device buffer sets",
    }


def run_also(args, name):
    """Secondary workload on the same GPU (context for the headline line)."""
    # about a second of timed work each: a video layer is ~50x a FLUX-2K layer, FLUX-4K ~4x
    steps = {"wan_video": max(10, args.steps // 50), "flux4k": max(20, args.steps // 16)}.get(name, max(50, args.steps // 4))
    sub = argparse.Namespace(**{**vars(args), "workload": name, "no_e2e": True, "no_extra": True, "steps": steps})
    r = run_ours(sub, 1, 0, int(os.environ.get("LOCAL_RANK", "0")))
    return {k: r[k] for k in ("value", "ms_per_step", "config", "roofline", "hbm_kernels", "gpu_launches",
                               "l2_flushed") if r.get(k) is not None}


# ----------------------------------------------------------------- oracle (CPU)


def cpu_oracle_sample(wl, budget_s: float, max_units: int | None = None):
    """Time the float64 oracle on (head, window) units of the workload: pooling of
    the head plus attention of one window's queries; returns (TFLOP/s, units, seconds, threads)."""
    from oracle import basa_oracle as O

    try:
        from threadpoolctl import threadpool_info

        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        threads = 1
    geo = O.Geometry(grid=wl.grid, window=wl.window, shift=wl.shift, pool=wl.pool, n_text=wl.n_text, routed_k=wl.routed_k)
    q, k, v = synth.make_inputs(wl, seed=0, heads=[0])
    q64, k64, v64 = (t.to(torch.float32).numpy().astype(np.float64) for t in (q, k, v))
    cnt = accounting.workload_counts(wl)
    flops_per_unit = cnt["attn_flops"] / (wl.B * wl.heads * cnt["n_win"])
    win = O.window_of_token(geo)
    units, t0 = 0, time.perf_counter()
    route = O.route_windows(q64, k64, geo)[0] if geo.routed_k else None
    kp, vp = O.pool_kv(k64, v64, geo) if geo.has_pool else (None, None)
    while True:
        w = units % cnt["n_win"]
        if w == 0 and units > 0 and geo.has_pool:
            kp, vp = O.pool_kv(k64, v64, geo)
        toks = np.nonzero(win == w)[0]
        O.attention_rows(q64, k64, v64, geo, 0, 0, toks, kp=kp, vp=vp, route_idx=route)
        units += 1
        el = time.perf_counter() - t0
        if el >= budget_s or (max_units and units >= max_units):
            break
    return units * flops_per_unit / el / 1e12, units, el, threads


def host_cpu():
    """(logical CPUs this process may use, CPU model name)."""
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        n = os.cpu_count() or 1
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return n, model


def cpu_baseline(args):
    """The oracle on the host: one BLAS thread, then all of them (numpy's pool)."""
    from threadpoolctl import threadpool_limits

    wl = synth.WORKLOADS[args.workload]
    nproc, model = host_cpu()
    with threadpool_limits(limits=1):
        t1, u1, e1, _ = cpu_oracle_sample(wl, args.cpu_budget / 3)
    tn, un, en, threads = cpu_oracle_sample(wl, args.cpu_budget)
    return {
        "value": round(tn, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
        "single_thread_value": round(t1, 6),
        "nproc": nproc, "cpu_model": model,
        "sample": f"{un} (head, window) units of {args.workload}, head 0, {en:.1f} s on {threads} BLAS threads "
                  f"(single thread: {u1} units, {e1:.1f} s), float64 numpy",
    }


def run_reference(args, world, rank):
    if rank != 0:
        return None
    wl = synth.WORKLOADS[args.workload]
    cnt = accounting.workload_counts(wl)
    per_step_budget = min(0.5, 150.0 / max(1, args.steps + args.warmup))
    cpu_oracle_sample(wl, 0.0, max_units=max(1, args.warmup))
    tflops, units, el, threads = cpu_oracle_sample(wl, per_step_budget * args.steps)
    step_ms = el / max(1, args.steps) * 1e3
    sample = f"{units} (head, window) units of {args.workload} (head 0): oracle pooling + all queries of a window, float64 numpy"
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(tflops, 6),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(wl, world),
        "cpu_baseline": {"value": round(tflops, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample,
                         "nproc": host_cpu()[0], "cpu_model": host_cpu()[1]},
        "e2e": {"value": round(tflops, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="flux2k", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--part", default="layer", choices=["layer", "backward"],
                    help="layer: the forward layer (the metric); backward: only the bfloat16 backward of the "
                         "workload at the last shift of its cycle (a context figure, e.g. for profiling)")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="replicas: a full layer per GPU (weak scaling); heads: one layer's (batch, head) units "
                         "split over the GPUs (strong scaling)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the secondary workload")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle cpu_baseline leg")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, world, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    world, rank, local = dist_setup()
    if args.part == "backward":
        if rank == 0:
            print(json.dumps({"backward_bf16": run_backward_bf16(args, args.workload,
                                                                 synth.SHIFT_CYCLES[args.workload][-1])}), flush=True)
        return
    res = run_ours(args, world, rank, local)
    if rank == 0 and world == 1 and not args.no_cpu:
        res["cpu_baseline"] = cpu_baseline(args)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
