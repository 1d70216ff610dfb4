"""Throughput of the W4A8-FP8 routed MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--experts w4a8|w8a8|nvfp4|hybrid] [--no-extra] [--no-cpu-baseline]

One step = one moe_w4a8_forward over a T-token batch (routing, FP8 quantization, grouped
gate/up GEMM, SwiGLU requantization, grouped down GEMM, shared experts if any, combine), with
inputs already in HBM.  The headline line times the largest config, prefill_t16384_shared
(16,384 tokens, uniform routing, 2 bf16 shared experts), for K steps; the other full-size
configs (decode_t8, decode_t64, prefill_t2048_zipf) follow under "workloads", each timed over
at least 200 ms of steps on the same layer.  `--experts` picks the routed-expert format
(row-scaled FP8, NVFP4, or NVFP4 hot + W4A8 cold experts instead of W4A8).  Batches rotate over
8 distinct seeded token sets, so the experts a step touches change from step to step; the
touched expert weights of one step (~0.57 GB at T=8) already exceed the 126 MB L2.  Ranks
(torchrun) are independent replicas, each with its own batches: weak scaling, no data-path
collective.

`--impl reference` times the CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import re
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s; % HBM roofline (decode) / % FP8 TC peak (prefill)"
HEADLINE = "prefill_t16384_shared"    # the largest config: the headline line
DEFAULT_WORKLOAD = HEADLINE
# the other configs of the benchmark, reported under "workloads" (the tiny config is parity-only)
EXTRA_WORKLOADS = ("decode_t8", "decode_t64", "prefill_t2048_zipf")
MIN_TIMED_MS = 200.0
EP_WORKLOADS = ("decode_t8", "decode_t64", "prefill_t2048_zipf")   # timed on the expert-parallel path too
N_BATCHES = 8
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def expert_bytes(wl, fmt="w4a8"):
    """Algorithmic bytes of one routed expert: packed INT4 codes + bf16 group scales (W4A8), or
    E4M3 codes + fp32 row scales (W8A8)."""
    if fmt == "w8a8":
        gate = wl.N * wl.H + wl.N * 4
        down = wl.H * wl.N + wl.H * 4
    elif fmt == "nvfp4":             # E2M1 codes + E4M3 block-16 scales + fp32 scale2
        gate = wl.N * wl.H // 2 + wl.N * wl.H // 16 + 4
        down = wl.H * wl.N // 2 + wl.H * wl.N // 16 + 4
    else:
        gate = wl.N * wl.H // 2 + wl.N * (wl.H // wl.group) * 2
        down = wl.H * wl.N // 2 + wl.H * (wl.N // wl.group) * 2
    return 2 * gate, down            # (gate+up, down)


def flops_per_pair(wl):
    return 2 * wl.H * 2 * wl.N + 2 * wl.N * wl.H


def router_line(wl, T, ms, hbm, bf16, peak_kind):
    """The router GEMM (moe_router_logits), timed apart from the layer step: HBM-bound at decode
    (the bf16 router weight is read once), bf16-tensor-bound at prefill."""
    if is_prefill(wl):
        flops = 2.0 * T * wl.H * wl.E
        ach = flops / (ms / 1e3) / 1e12
        return {"ms": round(ms, 4), "bound": "tensor", "achieved": round(ach, 1), "peak": bf16,
                "unit": "TFLOP/s", "frac": round(ach / bf16, 4),
                "peak_source": f"{peak_kind} bf16_tflops"}
    nbytes = wl.E * wl.H * 2 + T * wl.H * 2 + T * wl.E * 4
    ach = nbytes / (ms / 1e3) / 1e9
    return {"ms": round(ms, 4), "bound": "hbm", "achieved": round(ach, 1), "peak": hbm,
            "unit": "GB/s", "frac": round(ach / hbm, 4), "peak_source": f"{peak_kind} hbm_gbs",
            "algorithmic_bytes": int(nbytes)}


def graph_time(call, n, stream):
    """Mean device time (ms) of call(0..n-1), the n calls captured in one CUDA graph and replayed
    once between CUDA events; falls back to an eager loop if capture fails.  Returns (ms, graph?)."""
    import torch
    for i in range(3):
        call(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                call(i)
        g.replay()
        torch.cuda.synchronize()
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / n
        del g
        return ms, True
    except Exception:
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(n):
            call(i)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n, False


def is_prefill(wl):
    """Prefill-sized batches: the router GEMM runs on the tensor cores from T >= 256 and is
    scored against the bf16 peak here."""
    return wl.T >= 1024


KERNEL_SOURCES = {"w4a8": ("gemm_ws.cuh", "tc_pipe.cuh", "tc_ptx.cuh", "tc_tiles.cuh", "common.cuh"),
                  "w8a8": ("gemm_w8a8.cuh", "tc_pipe.cuh", "tc_ptx.cuh", "tc_tiles.cuh", "common.cuh"),
                  "nvfp4": ("gemm_nvfp4.cuh", "gemm_w8a8.cuh", "tc_pipe.cuh", "tc_ptx.cuh", "tc_tiles.cuh",
                            "common.cuh")}
PROFILE_FOR = {("w4a8", "decode_t8"): "gemm_w4a8_ws_decode_t8.md",
               ("w4a8", "prefill_t2048_zipf"): "gemm_w4a8_ws_prefill_t2048.md",
               ("w4a8", "prefill_t16384_shared"): "gemm_w4a8_ws_prefill_t16384.md",
               ("w8a8", "decode_t8"): "gemm_w8a8_decode_t8.md",
               ("w8a8", "prefill_t2048_zipf"): "gemm_w8a8_prefill_t2048.md",
               ("nvfp4", "decode_t8"): "gemm_nvfp4_decode_t8.md",
               ("nvfp4", "prefill_t2048_zipf"): "gemm_nvfp4_prefill_t2048.md"}


def ncu_traffic(workload, fmt="w4a8", algorithmic_bytes=None):
    """DRAM bytes per gate/up launch from the committed ncu summary of this workload, or None
    when there is none or the GEMM sources changed since it was taken.  A summary taken on a
    reduced-expert case of the same shape gives DRAM bytes per algorithmic byte instead, scaled
    here to this launch's algorithmic bytes (the traffic grows with the touched experts)."""
    name = PROFILE_FOR.get((fmt, workload))
    if not name:
        return None
    try:
        text = open(os.path.join(ROOT, "profiles", name)).read()
        vals = dict(re.findall(r"^\s*(traffic_gateup_bytes_per_launch|traffic_gateup_per_algorithmic_byte|"
                               r"sources_sha256):\s*(\S+)", text, flags=re.M))
        h = hashlib.sha256()
        for f in KERNEL_SOURCES[fmt]:
            with open(os.path.join(ROOT, "bit_quantized_moe_token_b200", "csrc", f), "rb") as fh:
                h.update(fh.read())
        if vals.get("sources_sha256") != h.hexdigest():
            return None
        if "traffic_gateup_bytes_per_launch" in vals:
            return int(vals["traffic_gateup_bytes_per_launch"])
        if algorithmic_bytes is not None and "traffic_gateup_per_algorithmic_byte" in vals:
            return int(float(vals["traffic_gateup_per_algorithmic_byte"]) * algorithmic_bytes)
        return None
    except (OSError, KeyError, ValueError):
        return None


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms by a background reader that
    stamps each line; summary(w) keeps the samples within 0.25 s of marked timed region w."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index):
        import threading
        self.idx, self.samples, self.proc = gpu_index, [], None
        self.windows = []
        self._lock = threading.Lock()
        self._thread = None

    def start(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return self
        self._thread = threading.Thread(target=self._read, daemon=True)
        self._thread.start()
        deadline = time.monotonic() + 5.0
        while time.monotonic() < deadline and not self.samples:
            time.sleep(0.02)
        return self

    def _read(self):
        for line in self.proc.stdout:
            with self._lock:
                self.samples.append((time.monotonic(), line.strip()))

    def mark_start(self):
        """Opens a timed window; returns its index."""
        self.windows.append([time.monotonic(), None])
        return len(self.windows) - 1

    def mark_end(self, w):
        self.windows[w][1] = time.monotonic()

    def stop(self):
        if not self.proc:
            return
        last = max((t1 for _, t1 in self.windows if t1 is not None), default=0.0)
        deadline = time.monotonic() + 1.0
        while time.monotonic() < deadline:
            with self._lock:
                if self.samples and self.samples[-1][0] > last:
                    break
            time.sleep(0.02)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()

    def summary(self, w):
        if w is None or w >= len(self.windows) or self.windows[w][1] is None:
            return None
        t0, t1 = self.windows[w]
        sm, mx, reasons = [], None, set()
        with self._lock:
            picked = [l for t, l in self.samples if t0 - 0.25 <= t <= t1 + 0.25]
        for l in picked:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for n, v in zip(self.NAMES, f[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "window_s": round(t1 - t0, 4)}


def replica_token_offset(rank, batch, T):
    """First token of batch `batch` on replica `rank`: the ranks draw disjoint stretches of the
    workload's token stream (weak scaling: every rank does a full batch per step)."""
    return (rank * N_BATCHES + batch) * T


def max_over_ranks(ms, device, world):
    """The slowest rank's device time (a single rank returns its own)."""
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world, T, steps, ms):
    """Tokens per second of all ranks together over `steps` steps of the slowest rank's `ms`."""
    return world * T * steps / (ms / 1e3)


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ------------------------------------------------------------------------------------------------
# our implementation
# ------------------------------------------------------------------------------------------------

class Formats:
    """The layer and its entry points for one routed-expert format, built once on the headline
    workload's weights (the configs share the same routed-expert draws; only the headline has
    shared experts, so the other configs take the same layer with the shared experts left out)."""

    def __init__(self, fmt, wl, dev):
        import torch
        import bit_quantized_moe_token_b200 as moe
        from bit_quantized_moe_token_b200.synthetic import (device_layer, device_layer_nvfp4,
                                                            device_layer_w8a8)
        self.moe, self.fmt = moe, fmt
        w8, f4, hy = fmt == "w8a8", fmt == "nvfp4", fmt == "hybrid"
        self.hot_set = set(synth.hot_experts(wl).tolist()) if hy else set()
        if hy:
            self.layer = moe.hybrid_from(device_layer(wl, device=dev), device_layer_nvfp4(wl, device=dev),
                                         synth.hot_experts(wl))
            torch.cuda.empty_cache()
        else:
            self.layer = (device_layer_w8a8 if w8 else device_layer_nvfp4 if f4 else device_layer)(wl, device=dev)
        self.fwd = (moe.moe_w8a8_forward if w8 else moe.moe_nvfp4_forward if f4 else moe.moe_hybrid_forward if hy
                    else moe.moe_w4a8_forward)
        self.fwd_profiled = (moe.moe_w8a8_forward_profiled if w8 else moe.moe_nvfp4_forward_profiled if f4
                             else moe.moe_hybrid_forward_profiled if hy else moe.moe_w4a8_forward_profiled)
        self.layout = (moe.moe_w8a8_workspace_layout if w8 else moe.moe_nvfp4_workspace_layout if f4
                       else moe.moe_hybrid_workspace_layout if hy else moe.moe_w4a8_workspace_layout)
        self.fwd_router = (moe.moe_w8a8_forward_router if w8 else moe.moe_nvfp4_forward_router if f4
                           else None if hy else moe.moe_w4a8_forward_router)
        self.kname = "W8A8" if w8 else "NVFP4" if f4 else "NVFP4-hot + W4A8-cold" if hy else "W4A8"
        self.dtype = ("e4m3 x e4m3 -> f32" if w8 else "f16(e2m1 x e4m3 scale) x f16(e4m3) -> f32" if f4
                      else "hot: f16(e2m1 x e4m3 scale) x f16(e4m3); cold: e4m3 x int4 -> f32" if hy
                      else "e4m3 x int4 -> f32")

    def layer_for(self, wl):
        if wl.n_shared:
            return self.layer
        import copy
        L = copy.copy(self.layer)
        tgt = L
        if self.fmt == "hybrid":
            L.cold = copy.copy(L.cold)
            tgt = L.cold
        tgt.sh_gate = tgt.sh_up = tgt.sh_down = None
        return L


def gateup_roofline(wl, fx, touched, touched_hot, steps, dom_ms, hbm, bf16, peak_kind):
    """Both bounds of the gate/up GEMM (the dominant kernel): its algorithmic bytes (touched
    experts' gate+up weights) over the measured HBM bandwidth, and its FLOPs over the dense FP8
    tensor peak (the measured bf16 cuBLAS peak x 2, NVIDIA's nominal FP8 / BF16 ratio).  The
    reported bound is the one with the longer ideal time; the other is given beside it."""
    T, k, fmt = wl.T, wl.k, fx.fmt
    mean_touched = sum(touched[i % N_BATCHES] for i in range(steps)) / steps
    if fmt == "hybrid":   # touched hot experts at NVFP4 bytes, the others at W4A8 bytes
        gu4, dn4 = expert_bytes(wl, "w4a8")
        guf, dnf = expert_bytes(wl, "nvfp4")
        mean_hot = sum(touched_hot[i % N_BATCHES] for i in range(steps)) / steps
        gu_bytes = (mean_hot * guf + (mean_touched - mean_hot) * gu4) / max(mean_touched, 1e-9)
        down_bytes = (mean_hot * dnf + (mean_touched - mean_hot) * dn4) / max(mean_touched, 1e-9)
    else:
        gu_bytes, down_bytes = expert_bytes(wl, fmt)
    dom_bytes = mean_touched * gu_bytes
    dom_flops = T * k * 2 * wl.H * 2 * wl.N
    fp8 = 2.0 * bf16
    t_hbm = dom_bytes / (hbm * 1e9)
    t_tc = dom_flops / (fp8 * 1e12)
    ach_gbs = dom_bytes / (dom_ms / 1e3) / 1e9
    ach_tf = dom_flops / (dom_ms / 1e3) / 1e12
    hbm_side = {"bound": "hbm", "achieved": round(ach_gbs, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(ach_gbs / hbm, 4), "peak_source": f"{peak_kind} hbm_gbs",
                "algorithmic_bytes_per_launch": int(dom_bytes),
                "units": f"{mean_touched:.1f} touched experts x {gu_bytes:.0f} B (gate+up codes+scales)"}
    tc_side = {"bound": "tensor", "achieved": round(ach_tf, 1), "peak": round(fp8, 1),
               "unit": "TFLOP/s", "frac": round(ach_tf / fp8, 4),
               "peak_source": f"{peak_kind} bf16_tflops x 2 (nominal FP8/BF16 ratio)",
               "algorithmic_flops_per_launch": int(dom_flops),
               "units": f"{T * k} routed pairs x {2 * wl.H * 2 * wl.N} FLOP (gate+up)"}
    main, other = (tc_side, hbm_side) if t_tc >= t_hbm else (hbm_side, tc_side)
    roofline = {"bound": main["bound"], "kernel": f"grouped gate/up {fx.kname} GEMM (stage)",
                "achieved": main["achieved"], "peak": main["peak"], "unit": main["unit"],
                "frac": main["frac"], "traffic": ncu_traffic(wl.name, fmt, dom_bytes)}
    roofline.update({k_: v for k_, v in main.items() if k_ not in roofline})
    roofline["other_bound"] = {k_: v for k_, v in other.items() if k_ != "units"}
    roofline["ideal_us"] = {"hbm": round(t_hbm * 1e6, 1), "tensor": round(t_tc * 1e6, 1)}
    roofline["launch_ms"] = round(dom_ms, 4)
    layer_bytes = mean_touched * (gu_bytes + down_bytes)
    return roofline, layer_bytes


def measure(fx, wl, steps, warmup, dev, stream, clk, rank, world, min_timed_ms=0.0, with_router=False):
    """One workload: warm-up, a stage-marked pass, the device-timed region (`steps` steps, or as
    many as make `min_timed_ms` when that is larger), the same steps end to end through the public
    entry point with host buffers, and optionally the router GEMM.  Every rank runs the same
    sequence of collectives (the max-over-ranks reductions)."""
    import torch
    import torch.distributed as dist
    moe = fx.moe
    layer = fx.layer_for(wl)
    T, k = wl.T, wl.k
    batches = [synth_batch(wl, rank, b, dev) for b in range(N_BATCHES)]
    out = torch.empty(T, wl.H, dtype=torch.bfloat16, device=dev)
    ws = moe.alloc_workspace(layer, T, k, dev)

    # touched experts per batch (for the algorithmic byte count), from the routing outputs
    lay = fx.layout(layer, T, k)
    touched, touched_hot = [], []
    for x, lg in batches:
        moe.forward(layer, x, lg, k, out=out, ws=ws)
        offs = ws[lay["expert_offsets"]:lay["expert_offsets"] + 4 * (wl.E + 1)].view(torch.int32)
        used = torch.nonzero(offs[1:] - offs[:-1] > 0).flatten().tolist()
        touched.append(len(used))
        touched_hot.append(sum(1 for e in used if e in fx.hot_set))
    torch.cuda.synchronize()
    if moe.moe_last_device_status() != 0:
        raise RuntimeError("device status: timeout during warm-up")
    for i in range(warmup):
        x, lg = batches[i % N_BATCHES]
        moe.forward(layer, x, lg, k, out=out, ws=ws)
    torch.cuda.synchronize()

    def make_events(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in evs:                 # torch creates the CUDA event on first record
            e.record(stream)
        return evs

    # stage breakdown: an untimed pass with every stage boundary marked
    full = [make_events(moe.N_STAGE_EVENTS) for _ in range(N_BATCHES)]
    torch.cuda.synchronize()
    for i in range(N_BATCHES):
        x, lg = batches[i]
        fx.fwd_profiled(layer, x, lg, k, out, ws, full[i])
    torch.cuda.synchronize()
    stage_ms = {s: 0.0 for s in moe.STAGES}
    for i in range(N_BATCHES):
        for j, s_ in enumerate(moe.STAGES):
            stage_ms[s_] += full[i][j].elapsed_time(full[i][j + 1]) / N_BATCHES

    # steps: at least `steps`, and enough for `min_timed_ms` of timed region (the largest count
    # over the ranks, so that every rank times the same number of steps)
    if min_timed_ms > 0:
        step_ms = sum(stage_ms.values())
        need = int(math.ceil(min_timed_ms / max(step_ms, 1e-3)))
        steps = max(steps, min(need, 20000))
        if world > 1:
            t = torch.tensor([steps], dtype=torch.int64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            steps = int(t.item())

    # ---- device-timed region: only the dominant kernel's boundaries are marked (2 events/step)
    DOM_A, DOM_B = 3, 4               # gate/up GEMM (stage boundaries, moe_w4a8.h)
    ev = []
    for _ in range(steps):
        pair = make_events(2)
        row = [None] * moe.N_STAGE_EVENTS
        row[DOM_A], row[DOM_B] = pair
        ev.append(row)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches = 0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    w = clk.mark_start()
    start.record(stream)
    # host enqueue time per step, over the first steps only: once the launch queue is full the
    # host waits for the GPU, and the figure would only repeat the device time
    n_host = min(steps, 16)
    h0 = time.perf_counter()
    for i in range(steps):
        x, lg = batches[i % N_BATCHES]
        launches += fx.fwd_profiled(layer, x, lg, k, out, ws, ev[i])
        if i + 1 == n_host:
            host_ms = (time.perf_counter() - h0) * 1e3 / n_host
    end.record(stream)
    torch.cuda.synchronize()
    clk.mark_end(w)
    if world > 1:
        dist.barrier()
    total_ms = start.elapsed_time(end)
    if moe.moe_last_device_status() != 0:
        raise RuntimeError("device status: timeout in the timed region")
    dom_ms = sum(ev[i][DOM_A].elapsed_time(ev[i][DOM_B]) for i in range(steps)) / steps
    total_ms = max_over_ranks(total_ms, dev, world)
    del ev

    # ---- end to end through the public entry point with host buffers: every step copies its
    # inputs from pinned host memory and reads the output back, pipelined as a serving loop
    # would: step i + 1's inputs go up on one copy stream and step i's output comes down on
    # another while step i computes (device inputs and outputs double-buffered); the timed region
    # spans every copy and every forward of the K steps
    hx = [b[0].cpu().pin_memory() for b in batches]
    hl = [b[1].cpu().pin_memory() for b in batches]
    hout = torch.empty(T, wl.H, dtype=torch.bfloat16).pin_memory()
    dx = [torch.empty_like(batches[0][0]) for _ in range(2)]
    dl = [torch.empty_like(batches[0][1]) for _ in range(2)]
    dout = [torch.empty_like(out) for _ in range(2)]
    up_s, down_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    ev_up, ev_fwd, ev_down = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def e2e_loop(n, e_start=None, e_end=None):
        if e_start is not None:
            e_start.record(stream)
        up_s.wait_stream(stream)
        down_s.wait_stream(stream)

        def upload(i):
            b = i % 2
            with torch.cuda.stream(up_s):
                if i >= 2:
                    up_s.wait_event(ev_fwd[b])          # forward i - 2 has read dx[b], dl[b]
                dx[b].copy_(hx[i % N_BATCHES], non_blocking=True)
                dl[b].copy_(hl[i % N_BATCHES], non_blocking=True)
                ev_up[b].record(up_s)
        upload(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                upload(i + 1)
            stream.wait_event(ev_up[b])
            if i >= 2:
                stream.wait_event(ev_down[b])           # step i - 2's output has left dout[b]
            fx.fwd(layer, dx[b], dl[b], k, dout[b], ws)
            ev_fwd[b].record(stream)
            with torch.cuda.stream(down_s):
                down_s.wait_event(ev_fwd[b])
                hout.copy_(dout[b], non_blocking=True)
                ev_down[b].record(down_s)
        if e_end is not None:
            e_end.record(down_s)                        # after the last read-back, hence after all
        stream.wait_stream(down_s)
        stream.wait_stream(up_s)

    e2e_loop(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e2e_loop(steps, e0, e1)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev, world)

    hbm, bf16, peak_kind = peaks()
    roofline, layer_bytes = gateup_roofline(wl, fx, touched, touched_hot, steps, dom_ms, hbm, bf16, peak_kind)
    tokens = world * T * steps
    r = {
        "value": round(whole_job_rate(world, T, steps, total_ms), 1), "unit": "tokens/s",
        "steps": steps, "timed_ms": round(total_ms, 3), "ms_per_step": round(total_ms / steps, 4),
        "host_enqueue_ms_per_step": round(host_ms, 4),
        "config": {"workload": wl.name, "experts": fx.fmt, "T": T, "H": wl.H, "N": wl.N, "E": wl.E,
                   "k": k, "routing": wl.routing, "n_shared": wl.n_shared, "seed": wl.seed,
                   "batches": N_BATCHES, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2: touched expert weights per step "
                         f"{layer_bytes / 1e9:.2f} GB vs 126 MB L2; {N_BATCHES} rotating batches"},
        "layer_hbm_gbs": round(layer_bytes / (total_ms / steps / 1e3) / 1e9, 1),
        "roofline": roofline,
        "stages_ms": {s_: round(v, 4) for s_, v in stage_ms.items()},
        "gpu_launches": launches,
        "e2e": {"value": round(tokens / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": T * wl.H * 2 + T * wl.E * 4,
                "d2h_bytes_per_step": T * wl.H * 2,
                "copies": "every step's inputs up from pinned host memory and its output back, on two "
                          "copy streams overlapping the neighbouring steps' forwards"},
        "clocks": clk.summary(w),
    }
    if with_router:
        r.update(router_timing(fx, wl, layer, batches, out, ws, steps, dev, stream, world, hbm, bf16, peak_kind))
    if moe.moe_last_device_status() != 0:
        raise RuntimeError("device status: timeout")
    return r


def synth_batch(wl, rank, b, dev):
    from bit_quantized_moe_token_b200.synthetic import device_inputs
    return device_inputs(wl, device=dev, t0=replica_token_offset(rank, b, wl.T), T=wl.T)


def router_timing(fx, wl, layer, batches, out, ws, steps, dev, stream, world, hbm, bf16, peak_kind):
    """Router logits (the step upstream of the layer's given logits), timed on its own: `steps`
    calls captured in one CUDA graph, so that the host-side cost of a Python call per tiny launch
    is not what is measured (an eager loop is the fallback if capture fails); then the whole
    layer fed by the router weight."""
    import torch
    moe = fx.moe
    T, k = wl.T, wl.k
    wr = torch.empty(wl.E, wl.H, dtype=torch.int16, device=dev)
    synth.dev_weight(wl.seed, synth.ROUTER_STREAM, wr, sigma=1.0 / math.sqrt(wl.H))
    wr = wr.view(torch.bfloat16)
    rlog = torch.empty(T, wl.E, dtype=torch.float32, device=dev)
    rids = torch.empty(T, k, dtype=torch.int32, device=dev)
    rgw = torch.empty(T, k, dtype=torch.float32, device=dev)
    rws = torch.empty(max(256, moe.moe_router_topk_workspace_bytes(T, wl.E, k)), dtype=torch.uint8, device=dev)
    n = min(steps, 200)
    r_ms, r_graph = graph_time(lambda i: moe.moe_router_logits(batches[i % N_BATCHES][0], wr, rlog), n, stream)
    rt_ms, _ = graph_time(lambda i: moe.moe_router_topk(batches[i % N_BATCHES][0], wr, k, rlog, rids, rgw, rws),
                          n, stream)
    r_ms = max_over_ranks(r_ms, dev, world)
    rt_ms = max_over_ranks(rt_ms, dev, world)
    lr_ms = None
    if fx.fwd_router is not None:
        for i in range(3):
            fx.fwd_router(layer, batches[i % N_BATCHES][0], wr, k, out, ws)
        q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        q0.record(stream)
        for i in range(n):
            fx.fwd_router(layer, batches[i % N_BATCHES][0], wr, k, out, ws)
        q1.record(stream)
        torch.cuda.synchronize()
        lr_ms = q0.elapsed_time(q1) / n
    lr_ms = max_over_ranks(lr_ms if lr_ms is not None else 0.0, dev, world)
    return {"router": dict(router_line(wl, T, r_ms, hbm, bf16, peak_kind), topk_fused_ms=round(rt_ms, 4),
                           cuda_graph=r_graph),
            "layer_with_router": None if lr_ms <= 0 else {
                "ms_per_step": round(lr_ms, 4), "value": round(world * T / (lr_ms / 1e3), 1),
                "unit": "tokens/s",
                "note": "moe_*_forward_router: router logits + the layer per step; routing follows "
                        "the synthetic N(0, 1/H) router weight (near uniform), not the workload's "
                        "given (e.g. Zipf) logits"}}


def ep_timing(fx, wl, steps, warmup, dev, stream, world, fused_ms):
    """The expert-parallel path (bit_quantized_moe_token_b200/ep.py) on this workload: experts split
    over the `world` ranks, each rank's own tokens dispatched to the owners and combined back.  With
    one rank the exchanges are skipped and what is timed is the path's own cost (records packed and
    unpacked, output rows put back in record order, the host read of the counts) against the fused
    forward's `fused_ms`."""
    import torch
    from bit_quantized_moe_token_b200.ep import EpLayer, local_experts
    layer = fx.layer_for(wl)
    rank = torch.distributed.get_rank() if world > 1 else 0
    ep = EpLayer(layer, local_experts(layer, rank, world))
    batches = [synth_batch(wl, rank, b, dev) for b in range(N_BATCHES)]
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device=dev)
    for i in range(max(warmup, 3)):
        x, lg = batches[i % N_BATCHES]
        ep.forward(x, lg, wl.k, out=out)
    n = max(steps, 20)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(n):
        x, lg = batches[i % N_BATCHES]
        ep.forward(x, lg, wl.k, out=out)
    e1.record(stream)
    torch.cuda.synchronize()
    if fx.moe.moe_last_device_status() != 0:
        raise RuntimeError("device status: error in the expert-parallel path")
    ms = max_over_ranks(e0.elapsed_time(e1) / n, dev, world)
    return {"n_ranks": world, "steps": n, "ms_per_step": round(ms, 4),
            "value": round(whole_job_rate(world, wl.T, n, ms * n), 1), "unit": "tokens/s",
            "fused_forward_ms_per_step": round(fused_ms, 4),
            "records_per_step": world * wl.T * wl.k}


def run_ours(args):
    import torch
    import torch.distributed as dist

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    wl = synth.WORKLOADS[args.workload]
    stream = torch.cuda.current_stream(dev)
    # the layer is built on the shared-expert config's weights (the same routed draws as every
    # full-size config); a config of other shapes (the tiny one) builds its own
    hw = synth.WORKLOADS[HEADLINE]
    same = (wl.E, wl.H, wl.N, wl.seed) == (hw.E, hw.H, hw.N, hw.seed)
    fx = Formats(args.experts, hw if same else wl, dev)
    clk = ClockSampler(local).start()
    head = measure(fx, wl, args.steps, args.warmup, dev, stream, clk, rank, world,
                   with_router=not args.no_router)
    extra = {}
    if not args.no_extra:
        for name in EXTRA_WORKLOADS:
            if name == wl.name:
                continue
            xw = synth.WORKLOADS[name]
            extra[name] = measure(fx, xw, args.steps, args.warmup, dev, stream, clk, rank, world,
                                  min_timed_ms=MIN_TIMED_MS)
            del extra[name]["config"]["parallelism"]
    ep = {}
    if args.experts == "w4a8" and (world == 1 or args.ep):
        # the expert-parallel path on the decode and mid-size configs (one rank: the exchanges
        # are skipped; several ranks only on request, since they run NCCL all-to-all exchanges)
        for name in EP_WORKLOADS:
            ref = head if name == wl.name else extra.get(name)
            if ref is None:
                continue
            ep[name] = ep_timing(fx, synth.WORKLOADS[name], args.steps, args.warmup, dev, stream, world,
                                 ref["ms_per_step"])
    clk.stop()
    result = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": head["steps"], "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": fx.dtype, "data": "synthetic",
    }
    for key in ("config", "host_enqueue_ms_per_step", "layer_hbm_gbs", "roofline", "stages_ms",
                "gpu_launches", "router", "layer_with_router", "e2e", "clocks"):
        if key in head:
            result[key] = head[key]
    if extra:
        result["workloads"] = extra
        result["workloads_note"] = (f"the other configs on the same layer (shared experts left out), "
                                    f"each timed over >= {MIN_TIMED_MS:.0f} ms of steps")
    if ep:
        result["expert_parallel"] = ep
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, fmt=args.experts)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# ------------------------------------------------------------------------------------------------
# the CPU oracle
# ------------------------------------------------------------------------------------------------

def oracle_sample(wl, t0, max_tokens, fmt="w4a8"):
    """A bounded sample of the workload for the CPU oracle: the first tokens of one batch,
    with the experts they route to packed (untimed setup)."""
    import oracle
    n = min(wl.T, max_tokens)
    x = synth.tokens(wl, t0, n)
    lg = synth.logits(wl, t0, n)
    ids, _ = oracle.route_topk(lg, wl.k)
    used = sorted(set(ids.reshape(-1).tolist()))
    if fmt == "w8a8":
        layer = oracle.quant_workload_layer_w8a8(wl, experts=used)
    elif fmt == "nvfp4":
        layer = oracle.quant_workload_layer_nvfp4(wl, experts=used)
    elif fmt == "hybrid":
        hot = synth.hot_experts(wl)
        cold_ids = np.array([e for e in range(wl.E) if e not in set(hot.tolist())], np.int32)
        w4 = oracle.pack_workload_layer(wl, experts=used)
        f4 = oracle.quant_workload_layer_nvfp4(wl, experts=used, with_shared=False)
        cold = oracle.Layer(len(cold_ids), wl.H, wl.N, w4.gate_packed[cold_ids], w4.up_packed[cold_ids],
                            w4.down_packed[cold_ids], w4.gate_scales[cold_ids], w4.up_scales[cold_ids],
                            w4.down_scales[cold_ids], group=wl.group, sh_gate=w4.sh_gate, sh_up=w4.sh_up,
                            sh_down=w4.sh_down)
        hotl = oracle.Layer.nvfp4(len(hot), wl.H, wl.N, f4.gate_f4[hot], f4.up_f4[hot], f4.down_f4[hot],
                                  f4.gate_bs[hot], f4.up_bs[hot], f4.down_bs[hot], f4.gate_s2[hot],
                                  f4.up_s2[hot], f4.down_s2[hot])
        layer = oracle.Layer.hybrid(cold, hotl, hot, cold_ids)
    else:
        layer = oracle.pack_workload_layer(wl, experts=used)
    return layer, x, lg, n


def cores_used():
    try:
        return int(os.environ.get("OMP_NUM_THREADS") or len(os.sched_getaffinity(0)))
    except Exception:
        return os.cpu_count() or 1


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def time_oracle(layer, x, lg, k, threads, reps=1):
    """Seconds per forward of the C oracle at `threads` OpenMP threads (packing not timed)."""
    import oracle
    oracle.set_threads(threads)
    t = time.perf_counter()
    for _ in range(reps):
        oracle.moe_forward(layer, x, lg, k)
    return (time.perf_counter() - t) / reps


def cpu_baseline(wl, fmt="w4a8", tokens_all=16, tokens_one=4):
    """The oracle as it stands on the host cores: a bounded sample of the workload (its first
    tokens, with the experts they route to packed beforehand), timed at all the process's cores
    and at one thread."""
    nproc = cores_used()
    layer, x, lg, n = oracle_sample(wl, 0, tokens_all, fmt)
    dt = time_oracle(layer, x, lg, wl.k, nproc)
    n1 = min(n, tokens_one)
    dt1 = time_oracle(layer, x[:n1], lg[:n1], wl.k, 1)
    import oracle
    oracle.set_threads(nproc)
    return {"value": round(n / dt, 3), "unit": "tokens/s", "cores": nproc, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{n} tokens of {wl.name}: one forward of the C oracle (fp32, OpenMP over experts "
                      f"and tokens) at {nproc} threads, {dt:.2f} s",
            "one_thread": {"value": round(n1 / dt1, 3), "unit": "tokens/s", "cores": 1,
                           "sample": f"{n1} tokens of {wl.name}, one forward at 1 thread, {dt1:.2f} s"}}


def run_reference(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        return
    wl = synth.WORKLOADS[args.workload]
    layer, x, lg, n = oracle_sample(wl, 0, args.ref_tokens, args.experts)
    nproc = cores_used()
    import oracle
    oracle.set_threads(nproc)
    for _ in range(args.warmup):
        oracle.moe_forward(layer, x, lg, wl.k)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle.moe_forward(layer, x, lg, wl.k)
    dt = time.perf_counter() - t
    value = n * args.steps / dt
    result = {
        "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": wl.name, "experts": args.experts, "T": wl.T, "H": wl.H, "N": wl.N,
                   "E": wl.E, "k": wl.k, "routing": wl.routing, "n_shared": wl.n_shared,
                   "seed": wl.seed, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": nproc,
                         "kind": "oracle", "cpu_model": cpu_model(),
                         "sample": f"{n} tokens of {wl.name} per step (C oracle, fp32)"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-tokens", type=int, default=8)
    ap.add_argument("--experts", default="w4a8", choices=["w4a8", "w8a8", "nvfp4", "hybrid"],
                    help="routed-expert weight format (default: W4A8 INT4 x FP8)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only --workload (not the other configs under \"workloads\")")
    ap.add_argument("--no-router", action="store_true", help="skip the router timings")
    ap.add_argument("--ep", action="store_true",
                    help="with several ranks, also time the expert-parallel path (NCCL all-to-all)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
