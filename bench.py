#!/usr/bin/env python
"""Throughput of the sparse MoE FFN block forward on B200.

One step = one whole forward pass of the block (router GEMM, top-k and
gates, offsets, permute, SwiGLU expert GEMMs, down GEMMs, combine with the
shared expert) over one batch of T tokens, through ``moe_forward`` of the C
ABI. Default workload: the DeepSeek-V3-shaped layer (T=4096, d=7168, 256
routed experts + 1 shared, inner 2048, top-8, sigmoid, 8 groups keep 4,
route_scale 2.5), bf16 storage with fp32 accumulation, synthetic seeded data.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl mine|reference]

With N > 1 (launched by torch.distributed.run) every rank runs an
independent replica on its own GPU (the block has no exchange step on one
node's data-parallel path): weak scaling, value = all ranks' tokens / the
slowest rank's time. Rank 0 prints one JSON line.

Besides the timed steps, the JSON line carries: the per-stage breakdown
(CUDA events between the stage entry points), the roofline of the dominant
kernel, the end-to-end rate through the public call with pinned host
buffers, the aux-loss-free balance step, the same routing with generic GELU
experts, the fused-permute variant, and the backward (recomputing, on saved
state, and a whole training step), each on the same inputs.

``--impl reference`` times the CPU oracle (the plain fp64 statement of the
block) on a bounded sample of the same workload: the reference arm.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "MoE-layer tokens/s and active TFLOP/s at DeepSeek-V3 shape; % bf16 / HBM roofline"
def kernels_per_forward(B, cfg, x) -> int:
    """Kernel launches of one moe_forward: the fused router (bf16, E <= 256)
    or router GEMM + top-k + chunk scan + offsets, then permute (left out
    when the router writes the row maps itself), gate/up, down and combine."""
    fused = cfg.dtype == "bf16" and cfg.E <= 256
    maps_in_route = B.moe_forward_gathers_rows(cfg, x) and B.moe_route_maps_supported(cfg)
    return (1 if fused else 4) + (3 if maps_in_route else 4)
CPU_SAMPLE_TOKENS = {"tiny_fp32": 64, "decode_fine": 32, "deepseek_v3": 16, "mixtral_8x7b": 8,
                     "deepseek_v3_skewed": 64}
REF_STEP_TOKENS = {"tiny_fp32": 64, "decode_fine": 8, "deepseek_v3": 2, "mixtral_8x7b": 2,
                   "deepseek_v3_skewed": 8}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="deepseek_v3")
    ap.add_argument("--impl", default="mine", choices=["mine", "reference"])
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of a CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--T", type=int, default=None, help="override the token count (profiling cases)")
    ap.add_argument("--E", type=int, default=None, help="override the routed expert count (profiling cases)")
    ap.add_argument("--f", type=int, default=None, help="override the expert inner width (profiling cases)")
    ap.add_argument("--forward-only", action="store_true",
                    help="stop after the timed forward steps and the stage breakdown (profiling runs)")
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="time the headline workload only (the others run at N=1 by default)")
    return ap.parse_args()


def workload(args):
    from mixture_experts_ffn_sigmoid_b200.inputs import CONFIGS
    cfg = CONFIGS[args.config]
    if args.T is not None or args.E is not None or args.f is not None:
        f = args.f or cfg.f
        cfg = cfg.with_(T=args.T or cfg.T, E=args.E or cfg.E, f=f,
                        f_shared=(f if cfg.f_shared else 0),
                        name=f"{cfg.name}_T{args.T or cfg.T}_E{args.E or cfg.E}" + (f"_f{f}" if args.f else ""))
    return cfg


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], tensor=d["bf16_tflops"], tensor_sustained=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, tensor=1590.0, tensor_sustained=1400.0, source="fallback")


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock, power and clock-event reasons sampled while work runs: from NVML
    every 20 ms when the library answers for this GPU, else from an `nvidia-smi`
    query loop every 100 ms. Both only read the GPU's state."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NVML_PERIOD_S = 0.02

    def __init__(self, device_index: int):
        self.samples = []
        self.proc = None
        self.dev = device_index
        self.source = None
        self._nvml = None
        self._stop_evt = None
        self.thread = None

    def _uuid(self):
        uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
        return uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"

    def _nvml_row(self):
        """One sample in the column order of FIELDS (reasons as Active / Not Active)."""
        n, h = self._nvml, self._handle
        sm = n.nvmlDeviceGetClockInfo(h, n.NVML_CLOCK_SM)
        mx = n.nvmlDeviceGetMaxClockInfo(h, n.NVML_CLOCK_SM)
        watts = n.nvmlDeviceGetPowerUsage(h) / 1000.0
        mask = n.nvmlDeviceGetCurrentClocksEventReasons(h)
        bits = (n.nvmlClocksEventReasonHwSlowdown, n.nvmlClocksEventReasonHwThermalSlowdown,
                n.nvmlClocksEventReasonSwThermalSlowdown, n.nvmlClocksEventReasonSwPowerCap)
        try:   # the memory clock, when this NVML reports it
            mem = n.nvmlDeviceGetClockInfo(h, n.NVML_CLOCK_MEM)
        except Exception:
            mem = ""
        return [str(sm), str(mx), f"{watts:.2f}", hex(mask)] + \
            ["Active" if mask & b else "Not Active" for b in bits] + [str(mem)]

    def _start_nvml(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._handle = pynvml.nvmlDeviceGetHandleByUUID(self._uuid())
            self.samples.append((time.time(), self._nvml_row()))   # the first read must work
        except Exception:
            self._shutdown_nvml()
            self.samples = []
            return False
        self._stop_evt = threading.Event()
        self.thread = threading.Thread(target=self._poll_nvml, daemon=True)
        self.thread.start()
        self.source = "nvml"
        return True

    def _poll_nvml(self):
        while not self._stop_evt.wait(self.NVML_PERIOD_S):
            try:
                self.samples.append((time.time(), self._nvml_row()))
            except Exception:
                return

    def _shutdown_nvml(self):
        if self._nvml is not None:
            try:
                self._nvml.nvmlShutdown()
            except Exception:
                pass
            self._nvml = None

    def start(self):
        if self._start_nvml():
            return
        try:
            sel = self._uuid()
        except Exception:
            sel = str(self.dev)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", sel, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.source = "nvidia-smi"
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [v.strip() for v in line.split(",")]))

    def stop(self):
        if self._stop_evt is not None:
            self._stop_evt.set()
            if self.thread is not None:
                self.thread.join(timeout=2)
            self._shutdown_nvml()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = [s for t, s in self.samples if t0 <= t <= t1]
        window = "timed region"
        if len(rows) < 3:
            rows = [s for _, s in self.samples]
            window = "warm-up and timed region (timed region shorter than 3 samples)"
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[0]) for r in rows if num(r[0]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if len(r) > 4 + i and r[4 + i] == "Active"})
        mem = [num(r[8]) for r in rows if len(r) > 8 and num(r[8]) is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": num(rows[0][1]), "reasons": reasons, "samples": len(rows), "window": window,
                "source": self.source, "power_w_max": max((num(r[2]) or 0.0) for r in rows),
                "mem_mhz": statistics.median(mem) if mem else None}


# ------------------------------------------------------- multi-rank timing
def reduce_max(value: float, device, world: int) -> float:
    """The slowest rank's value: every rank contributes, every rank gets the max."""
    if world <= 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.item()


def whole_job_rate(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Tokens per second of all ranks together (each rank runs its own replica)."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


# ------------------------------------------------------------ work accounting
def stage_work(cfg, counts, gather=False):
    """Algorithmic bytes (compulsory HBM traffic) and flops of each stage for one forward.
    gather: the gate/up GEMM reads token rows from x itself and the permute
    writes the maps only (moe_forward_gathers_rows)."""
    es = cfg.elem_bytes
    T, d, E, k, f, fs = cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.f_shared
    touched = int((counts > 0).sum())
    rows, srows = T * k, (T if fs else 0)
    w = {}
    # route: x and the router read, the summed fp32 logits written once (kept
    # for the backward pass), indices and gates written.
    w["route"] = dict(bytes=(T * d + E * d) * es + T * k * 8 + T * E * 4, flops=2.0 * T * E * d)
    w["permute"] = dict(bytes=(0 if gather else (T * d + rows * d) * es) + rows * 8 + T * k * 4, flops=0.0)
    w["gate_up"] = dict(bytes=(touched * 2 * f * d + 2 * fs * d) * es + (rows * d + srows * d) * es
                        + (rows * f + srows * fs) * es,
                        flops=4.0 * (rows * f + srows * fs) * d)
    w["down"] = dict(bytes=(touched * d * f + d * fs) * es + (rows * f + srows * fs) * es
                     + (rows * d + srows * d) * es,
                     flops=2.0 * (rows * f + srows * fs) * d)
    w["combine"] = dict(bytes=(rows * d + srows * d + T * d) * es + rows * 8, flops=0.0)
    return w, touched


def source_sha(paths):
    """First 16 hex digits of the sha256 of the files' contents, in order."""
    h = hashlib.sha256()
    for path in ([paths] if isinstance(paths, str) else paths):
        h.update(open(path, "rb").read())
    return h.hexdigest()[:16]


def traffic_for(workload, stage):
    """DRAM bytes per launch from a committed ncu summary, if the kernel is unchanged."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d.get(workload, {}).get(stage)
        if not e:
            return None
        srcs = e["sources"] if "sources" in e else [e["source"]]
        if source_sha([os.path.join(ROOT, x) for x in srcs]) != e["source_sha256_16"]:
            return None
        return e["bytes_per_launch"]
    except Exception:
        return None


def measure_gelu_experts(B, cfg, inp, counts, stream, reps):
    """moe_forward_gelu (generic experts W2 GELU(W1 u + b1) + b2, no shared
    expert) on this workload's x, router and w1/w2, timed over a CUDA graph."""
    from mixture_experts_ffn_sigmoid_b200.inputs import make_expert_biases
    gcfg = cfg.with_(f_shared=0)
    dev = inp["x"].device
    bb = make_expert_biases(gcfg, dev)
    ws_g = B.alloc_workspace(gcfg, dev)
    yg = torch.empty((cfg.T, cfg.d), dtype=cfg.torch_dtype, device=dev)

    def fwd():   # on the current stream, so that the graph below captures it
        B.moe_forward_gelu(gcfg, inp["x"], inp["w_router"], inp["bias"], inp["w1"], bb["b1"], inp["w2"],
                           bb["b2"], yg, ws_g)

    for _ in range(3):
        fwd()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fwd()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    del g
    assert B.moe_get_device_error(ws_g) == B.MOE_OK
    ms = e0.elapsed_time(e1) / reps
    es = cfg.elem_bytes
    T, d, E, k, f = cfg.T, cfg.d, cfg.E, cfg.k, cfg.f
    touched = int((counts > 0).sum())
    flops = 2.0 * T * (E * d + k * 2 * d * f)
    weight_bytes = touched * 2 * f * d * es + touched * (f + d) * 4
    return {"workload": f"{cfg.name} routed experts as GELU FFNs with b1/b2 (no shared expert)",
            "ms_per_step": ms, "tokens_per_s": T / (ms / 1e3),
            "active_tflops": flops / (ms / 1e3) / 1e12,
            "expert_weight_gbs": weight_bytes / (ms / 1e3) / 1e9, "graph_replays": reps}


def backward_work(cfg, touched):
    """Algorithmic flops and HBM bytes of one moe_backward call.

    Flops: the router (logits, input and weight gradients: 3 x 2TEd) and, per
    routed row (T k of them) and shared row (T), the recomputed
    pre-activations (2 x 2df), dh' (2df), dx (2 x 2df) and the three weight
    gradients (3 x 2df): 16 d f per row. Bytes: every touched expert's W1, W3
    read twice (pre-activations, dx) and W2 once; every weight gradient
    written once (untouched experts' as zeros); x and dy read, dx written.
    """
    es = cfg.elem_bytes
    T, d, E, k, f, fs = cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.f_shared
    flops = 6.0 * T * E * d + 16.0 * d * (T * k * f + T * fs)
    w_read = (touched * 5 * f * d + 5 * fs * d + E * d) * es
    g_write = (E * 3 * f * d + 3 * fs * d + E * d) * es
    act = 3 * T * d * es
    return flops, w_read + g_write + act


def measure_backward(B, cfg, inp, touched, stream, reps):
    """moe_backward (routing and pre-activations recomputed, every gradient
    written) timed over a CUDA graph on the workload's inputs and a seeded dy."""
    dev = inp["x"].device
    dt = cfg.torch_dtype
    g = torch.Generator(device=dev)
    g.manual_seed(9)
    dy = torch.randn((cfg.T, cfg.d), generator=g, device=dev).to(dt)
    sh = cfg.f_shared > 0
    outs = [torch.empty((cfg.T, cfg.d), dtype=dt, device=dev), torch.empty((cfg.E, cfg.d), dtype=dt, device=dev),
            torch.empty((cfg.E, cfg.f, cfg.d), dtype=dt, device=dev),
            torch.empty((cfg.E, cfg.f, cfg.d), dtype=dt, device=dev),
            torch.empty((cfg.E, cfg.d, cfg.f), dtype=dt, device=dev),
            torch.empty((cfg.f_shared, cfg.d), dtype=dt, device=dev) if sh else None,
            torch.empty((cfg.f_shared, cfg.d), dtype=dt, device=dev) if sh else None,
            torch.empty((cfg.d, cfg.f_shared), dtype=dt, device=dev) if sh else None]
    wsb = B.alloc_backward_workspace(cfg, dev)

    def bwd():   # on the current stream, so that the graph below captures it
        B.moe_backward(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w1"], inp["w3"], inp["w2"], inp["ws1"],
                       inp["ws3"], inp["ws2"], dy, *outs, wsb)

    for _ in range(2):
        bwd()
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        bwd()
    gr.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        gr.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    del gr
    assert B.moe_get_device_error(wsb) == B.MOE_OK
    ms = e0.elapsed_time(e1) / reps
    flops, nbytes = backward_work(cfg, touched)

    # Training step: moe_forward_train keeps routing and pre-activations in the
    # workspace, moe_backward_saved uses them (no recomputation).
    y = torch.empty((cfg.T, cfg.d), dtype=dt, device=dev)

    def fwd_train():
        B.moe_forward_train(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w1"], inp["w3"], inp["w2"],
                            inp["ws1"], inp["ws3"], inp["ws2"], y, wsb)

    def bwd_saved():
        B.moe_backward_saved(cfg, inp["x"], inp["w_router"], inp["w1"], inp["w3"], inp["w2"], inp["ws1"],
                             inp["ws3"], inp["ws2"], dy, *outs, wsb)

    def timed(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        gg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gg):
            fn()
        gg.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            gg.replay()
        b.record(stream)
        torch.cuda.synchronize()
        del gg
        assert B.moe_get_device_error(wsb) == B.MOE_OK
        return a.elapsed_time(b) / reps

    fwd_train()
    saved_ms = timed(bwd_saved)
    step_ms = timed(lambda: (fwd_train(), bwd_saved()))
    del outs, wsb
    return {"ms_per_step": ms, "tokens_per_s": cfg.T / (ms / 1e3), "tflops": flops / (ms / 1e3) / 1e12,
            "gbs": nbytes / (ms / 1e3) / 1e9, "algorithmic_flops": flops, "algorithmic_bytes": nbytes,
            "graph_replays": reps,
            "note": "recomputes routing and SwiGLU pre-activations; writes dx and every weight gradient",
            "saved_ms": saved_ms,
            "train_step_ms": step_ms,
            "train_step_note": "moe_forward_train + moe_backward_saved (pre-activations kept from the forward)"}


def measure_fused_permute(B, cfg, inp, idx, offsets, perm_src, inv_row, h, h_s, ws, stream, reps):
    """The permute fused into the gate/up GEMM: maps-only permute, then the
    GEMM gathering token rows from x (cp.async gather warps). Same h bytes as
    the packed chain; timed with events like the stage breakdown."""
    h2 = torch.empty_like(h)
    hs2 = torch.empty_like(h_s) if h_s is not None else None
    calls = [lambda: B.moe_permute(cfg, None, idx, offsets, None, perm_src, inv_row, ws),
             lambda: B.moe_expert_gate_up_gather(cfg, inp["x"], perm_src, offsets, inp["w1"], inp["w3"],
                                                 inp["ws1"], inp["ws3"], h2, hs2, ws)]
    for _ in range(2):
        for c in calls:
            c()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
    for i in range(reps):
        evs[i][0].record(stream)
        for j, c in enumerate(calls):
            c()
            evs[i][j + 1].record(stream)
    torch.cuda.synchronize()
    assert torch.equal(h2, h), "gathered and packed gate/up disagree"
    pm = statistics.mean(evs[i][0].elapsed_time(evs[i][1]) for i in range(reps))
    gm = statistics.mean(evs[i][1].elapsed_time(evs[i][2]) for i in range(reps))
    return {"permute_maps_ms": pm, "gate_up_gather_ms": gm, "fused_ms": pm + gm,
            "note": "moe_forward gathers only with single-CTA token tiles (under 128 rows); "
                    "this shape runs CTA pairs, where the packed copy plus gate/up is faster"}


def layer_bytes(cfg, touched):
    """The layer's own compulsory HBM bytes for one forward: x, the router
    matrix (and bias), every touched expert's three matrices, the shared
    expert's, and y. Intermediates of this implementation are not counted."""
    es = cfg.elem_bytes
    T, d, E, f, fs = cfg.T, cfg.d, cfg.E, cfg.f, cfg.f_shared
    return (2 * T * d + E * d + touched * 3 * f * d + 3 * fs * d) * es + (E * 4 if cfg.bias else 0)


def stage_breakdown(B, cfg, inp, ws, stream, n):
    """The forward through the per-stage entry points, captured once as a CUDA
    graph with a CUDA event recorded between consecutive stage calls (event
    nodes inside the graph), replayed n times; each replay is read back before
    the next. A stage's time is the device time between its events in a chain
    that runs like moe_forward's graph, once per pass. Returns the mean
    milliseconds per stage, the stage outputs (of the last pass), and each
    short stage's (route, permute, combine) milliseconds per call when its
    entry point runs back to back in a graph of its own (no event node
    between launches)."""
    dev = inp["x"].device
    T, d, E, k = cfg.T, cfg.d, cfg.E, cfg.k
    rows = T * k
    dt = cfg.torch_dtype
    sh = cfg.f_shared > 0
    o = dict(idx=torch.empty((T, k), dtype=torch.int32, device=dev),
             gate=torch.empty((T, k), dtype=torch.float32, device=dev),
             counts=torch.empty((E,), dtype=torch.int32, device=dev),
             offsets=torch.empty((E + 1,), dtype=torch.int32, device=dev),
             x_perm=torch.empty((rows, d), dtype=dt, device=dev),
             perm_src=torch.empty((rows,), dtype=torch.int32, device=dev),
             inv_row=torch.empty((T, k), dtype=torch.int32, device=dev),
             h=torch.empty((rows, cfg.f), dtype=dt, device=dev),
             h_s=torch.empty((T, cfg.f_shared), dtype=dt, device=dev) if sh else None,
             y_perm=torch.empty((rows, d), dtype=dt, device=dev),
             y_s=torch.empty((T, d), dtype=dt, device=dev) if sh else None,
             y=torch.empty((T, d), dtype=dt, device=dev))
    names = ["route", "permute", "gate_up", "down", "combine"]
    # The same path moe_forward takes: packed rows, or (single-CTA token
    # tiles) the row maps only and the GEMM gathering rows from x; the maps
    # come from the router itself when the batch is one router tile (the
    # permute stage is then empty: the time between two adjacent events).
    gather = B.moe_forward_gathers_rows(cfg, inp["x"])
    maps_in_route = gather and B.moe_route_maps_supported(cfg)
    calls = [
        (lambda: B.moe_route_maps(cfg, inp["x"], inp["w_router"], inp["bias"], o["idx"], o["gate"], o["counts"],
                                  o["offsets"], o["perm_src"], o["inv_row"], ws)) if maps_in_route
        else (lambda: B.moe_route(cfg, inp["x"], inp["w_router"], inp["bias"], o["idx"], o["gate"], o["counts"],
                                  o["offsets"], ws)),
        None if maps_in_route
        else (lambda: B.moe_permute(cfg, None, o["idx"], o["offsets"], None, o["perm_src"], o["inv_row"], ws))
        if gather
        else (lambda: B.moe_permute(cfg, inp["x"], o["idx"], o["offsets"], o["x_perm"], o["perm_src"],
                                    o["inv_row"], ws)),
        (lambda: B.moe_expert_gate_up_gather(cfg, inp["x"], o["perm_src"], o["offsets"], inp["w1"], inp["w3"],
                                             inp["ws1"], inp["ws3"], o["h"], o["h_s"], ws)) if gather
        else (lambda: B.moe_expert_gate_up(cfg, o["x_perm"], o["offsets"], inp["w1"], inp["w3"],
                                           inp["x"] if sh else None, inp["ws1"], inp["ws3"], o["h"], o["h_s"], ws)),
        lambda: B.moe_expert_down(cfg, o["h"], o["offsets"], inp["w2"], o["h_s"], inp["ws2"], o["y_perm"],
                                  o["y_s"], ws),
        lambda: B.moe_combine(cfg, o["y_perm"], o["inv_row"], o["gate"], o["y_s"], o["y"]),
    ]
    for _ in range(2):
        for c in calls:
            if c:
                c()
    torch.cuda.synchronize()
    # external: recorded inside the capture as timing event nodes
    evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(calls) + 1)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        evs[0].record()
        for j, c in enumerate(calls):
            if c:
                c()
            evs[j + 1].record()
    g.replay()
    torch.cuda.synchronize()
    acc = [0.0] * len(calls)
    for _ in range(n):
        g.replay()
        torch.cuda.synchronize()
        for j in range(len(calls)):
            acc[j] += evs[j].elapsed_time(evs[j + 1])
    del g
    # The short stages alone: `reps` calls of the entry point back to back in
    # one CUDA graph (launches pipelined as inside moe_forward's graph, no
    # event node between them), device time per call. Every call redoes the
    # whole stage on the same inputs. The event nodes of the chain above add
    # a few microseconds per stage, which is a large share of these; the
    # expert GEMMs are left out (eight of them back to back run under the
    # power cap, below the clock they run at in the step).
    reps = 8
    iso = {}
    for j, c in enumerate(calls):
        if names[j] not in ("route", "permute", "combine"):
            continue
        if c is None:   # no launch of its own on this path
            iso[names[j]] = 0.0
            continue
        gj = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gj):
            for _ in range(reps):
                c()
        gj.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(2):
            gj.replay()
        e1.record()
        torch.cuda.synchronize()
        iso[names[j]] = e0.elapsed_time(e1) / (2 * reps)
        del gj
    assert B.moe_get_device_error(ws) == B.MOE_OK
    return {nm: acc[j] / n for j, nm in enumerate(names)}, o, iso


def graph_step_ms(B, cfg, inp, ws, y, stream, steps, warmup):
    """Milliseconds per moe_forward replayed from a CUDA graph, after warm-up."""
    def fwd():
        B.moe_forward(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w1"], inp["w3"], inp["w2"],
                      inp["ws1"], inp["ws3"], inp["ws2"], y, ws)

    for _ in range(max(warmup, 3)):
        fwd()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fwd()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    e0.record(stream)
    for _ in range(steps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    del g
    assert B.moe_get_device_error(ws) == B.MOE_OK
    return e0.elapsed_time(e1) / steps, t0, t1


def measure_workload(B, name, dev, stream, steps, warmup, sampler, peaks):
    """One more workload of the pages, on its own inputs: the CUDA-graph step,
    its stage times, and the fraction of the roof that binds it (HBM for the
    weight-streaming shapes, the sustained tensor peak for the expert GEMMs of
    the compute-bound ones), with the clock samples of its own timed region."""
    from mixture_experts_ffn_sigmoid_b200.inputs import CONFIGS, make_inputs
    cfg = CONFIGS[name]
    inp = make_inputs(cfg, dev, seed=0)
    ws = B.alloc_workspace(cfg, dev)
    y = torch.empty((cfg.T, cfg.d), dtype=cfg.torch_dtype, device=dev)
    ms, t0, t1 = graph_step_ms(B, cfg, inp, ws, y, stream, steps, warmup)
    stage_ms, o, stage_iso = stage_breakdown(B, cfg, inp, ws, stream, max(3, min(steps, 50)))
    assert torch.equal(o["y"], y), f"{name}: per-stage chain and moe_forward disagree"
    work, touched = stage_work(cfg, o["counts"].cpu(), B.moe_forward_gathers_rows(cfg, inp["x"]))
    expert_ms = stage_ms["gate_up"] + stage_ms["down"]
    expert_flops = work["gate_up"]["flops"] + work["down"]["flops"]
    expert_bytes = work["gate_up"]["bytes"] + work["down"]["bytes"]
    lb = layer_bytes(cfg, touched)
    flops = cfg.active_flops()
    r = {"config": {"T": cfg.T, "d": cfg.d, "E": cfg.E, "k": cfg.k, "f": cfg.f, "f_shared": cfg.f_shared,
                    "gate": "sigmoid" if cfg.gate_mode else "softmax", "n_groups": cfg.n_groups,
                    "topk_groups": cfg.topk_groups, "route_scale": cfg.route_scale, "dtype": cfg.dtype},
         "ms_per_step": ms, "steps": steps, "cuda_graph": True,
         "tokens_per_s": cfg.T / (ms / 1e3), "active_tflops": flops / (ms / 1e3) / 1e12,
         "experts_touched": touched, "stages_ms": stage_ms, "stages_ms_back_to_back": stage_iso,
         "layer_bytes": lb, "step_gbs": lb / (ms / 1e3) / 1e9,
         "step_frac_hbm": lb / (ms / 1e3) / 1e9 / peaks["hbm"],
         "expert_gemm": {"ms": expert_ms, "tflops": expert_flops / (expert_ms / 1e3) / 1e12,
                         "frac_tensor_sustained": expert_flops / (expert_ms / 1e3) / 1e12 / peaks["tensor_sustained"],
                         "gbs": expert_bytes / (expert_ms / 1e3) / 1e9,
                         "frac_hbm": expert_bytes / (expert_ms / 1e3) / 1e9 / peaks["hbm"]},
         "clocks": sampler.summary(t0, t1)}
    hbm_t = lb / (peaks["hbm"] * 1e9)
    tc_t = flops / (peaks["tensor_sustained"] * 1e12)
    if cfg.dtype != "bf16":
        r["binding_roof"] = "launch latency (parity-sized workload)"
    elif tc_t > hbm_t:
        r["binding_roof"] = "tensor"
        r["binding_frac"] = r["expert_gemm"]["frac_tensor_sustained"]
    else:
        r["binding_roof"] = "hbm"
        r["binding_frac"] = r["step_frac_hbm"]
    del inp, ws, y, o
    torch.cuda.empty_cache()
    return r


# ---------------------------------------------------------------- oracle arm
def oracle_sample_time(cfg, inp, n_tokens, seed):
    """Run the CPU oracle on ``n_tokens`` seeded tokens; returns (seconds, threads)."""
    import numpy as np
    import oracle.moe_oracle as orc
    from mixture_experts_ffn_sigmoid_b200.inputs import sample_token_ids

    def f64(t):
        return None if t is None else t.detach().to("cpu").to(torch.float64).numpy()

    class Lazy:
        def __init__(self, t):
            self.t = t

        def __getitem__(self, e):
            return f64(self.t[int(e)])

    tok = sample_token_ids(cfg.T, n_tokens, seed=seed)
    x = inp["x"][tok.to(inp["x"].device)]
    wr = f64(inp["w_router"])
    bias = f64(inp["bias"])
    shared = [f64(inp[k]) for k in ("ws1", "ws3", "ws2")]
    t0 = time.perf_counter()
    r = orc.route(f64(x), wr, bias, cfg.k, cfg.gate_mode, cfg.n_groups, cfg.topk_groups, cfg.route_scale)
    orc.expert_outputs(f64(x), r["idx"], r["gates"], Lazy(inp["w1"]), Lazy(inp["w3"]), Lazy(inp["w2"]),
                       *shared)
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        threads = os.cpu_count() or 1
    return dt, threads


def workload_config(cfg, world: int) -> dict:
    """The JSON line's `config`: the workload, identical on both arms."""
    return {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "E": cfg.E, "k": cfg.k, "f": cfg.f,
            "f_shared": cfg.f_shared, "gate": "sigmoid" if cfg.gate_mode else "softmax",
            "n_groups": cfg.n_groups, "topk_groups": cfg.topk_groups, "route_scale": cfg.route_scale,
            "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2: every step streams the layer's expert weights "
                  f"({(cfg.E * 3 * cfg.f * cfg.d + 3 * cfg.f_shared * cfg.d) * cfg.elem_bytes / 1e9:.2f} GB)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from mixture_experts_ffn_sigmoid_b200.inputs import make_inputs
    cfg = workload(args)
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0"))) if torch.cuda.is_available() \
        else torch.device("cpu")
    inp = make_inputs(cfg, dev, seed=0)
    n = min(REF_STEP_TOKENS.get(args.config, 4), cfg.T)
    for i in range(args.warmup):
        oracle_sample_time(cfg, inp, n, seed=100 + i)
    times, threads = [], 1
    for i in range(args.steps):
        dt, threads = oracle_sample_time(cfg, inp, n, seed=1000 + i)
        times.append(dt)
    total = sum(times)
    value = n * args.steps / total
    sample = f"{n} seeded tokens of the {cfg.name} workload per step (routing over all experts, " \
             f"FFN of every selected expert and the shared expert, fp64)"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(cfg, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- our arm
def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    from mixture_experts_ffn_sigmoid_b200 import binding as B
    from mixture_experts_ffn_sigmoid_b200.inputs import make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    cfg = workload(args)
    B.lib()
    inp = make_inputs(cfg, dev, seed=0)
    if rank > 0:
        inp["x"] = make_inputs(cfg, dev, seed=rank, x_only=True)["x"]
    T, d = cfg.T, cfg.d
    ws = B.alloc_workspace(cfg, dev)
    y = torch.empty((T, d), dtype=cfg.torch_dtype, device=dev)

    def forward():
        B.moe_forward(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w1"], inp["w3"], inp["w2"],
                      inp["ws1"], inp["ws3"], inp["ws2"], y, ws)

    sampler = ClockSampler(local)
    sampler.start()
    for _ in range(max(args.warmup, 3)):
        forward()
    torch.cuda.synchronize()
    assert B.moe_get_device_error(ws) == B.MOE_OK

    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            forward()
        graph.replay()
        torch.cuda.synchronize()
    run = graph.replay if graph is not None else forward

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    # ---- timed region: K whole forward passes --------------------------------
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    ev0.record(stream)
    for _ in range(args.steps):
        run()
    ev1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier()
    ms_total = reduce_max(ev0.elapsed_time(ev1), dev, world)
    ms_step = ms_total / args.steps
    value = whole_job_rate(T, world, ms_step)
    assert B.moe_get_device_error(ws) == B.MOE_OK
    clocks = sampler.summary(t_wall0, t_wall1)

    # ---- stage breakdown: the same kernels through the per-stage entry points,
    # one CUDA event between stages on the launching stream ----------------------
    k, E = cfg.k, cfg.E
    n_stage = max(3, min(args.steps, 50))
    names = ["route", "permute", "gate_up", "down", "combine"]
    stage_ms, so, stage_iso = stage_breakdown(B, cfg, inp, ws, stream, n_stage)
    idx, gate, counts, offsets = so["idx"], so["gate"], so["counts"], so["offsets"]
    perm_src, inv_row, h, h_s = so["perm_src"], so["inv_row"], so["h"], so["h_s"]
    assert torch.equal(so["y"], y), "per-stage chain and moe_forward disagree"
    if args.forward_only:
        sampler.stop()
        if rank == 0:
            print(json.dumps({"profiling_run": cfg.name, "ms_per_step": ms_step, "stages_ms": stage_ms,
                              "stages_ms_back_to_back": stage_iso,
                              "clocks": clocks}), flush=True)
        if graph is not None:
            del graph
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    # ---- the pages' other workloads (one GPU only): each on its own inputs,
    # CUDA-graph step, stage times, binding-roof fraction, its own clocks. They
    # run right after the headline's own timing, before the long backward and
    # end-to-end measurements heat the GPU. ---------------------------------------
    peaks = measured_peaks()
    extra = None
    if world == 1 and not args.no_extra_workloads and args.T is None and args.E is None and args.f is None:
        from mixture_experts_ffn_sigmoid_b200.inputs import CONFIGS
        extra = {}
        # Lightest first, each after a second of idle GPU: the power cap that a
        # heavy workload engages (sw_power_cap) then does not carry over into
        # the next one's clocks, which each line reports for its own window.
        for name in sorted((n for n in CONFIGS if n != cfg.name), key=lambda n: CONFIGS[n].active_flops()):
            torch.cuda.synchronize()
            time.sleep(1.0)
            extra[name] = measure_workload(B, name, dev, stream, max(3, min(args.steps, 50)), args.warmup,
                                           sampler, peaks)
    fused = measure_fused_permute(B, cfg, inp, idx, offsets, perm_src, inv_row, h, h_s, ws, stream,
                                  n_stage) if cfg.dtype == "bf16" else None
    if fused is not None:
        fused["packed_ms"] = stage_ms["permute"] + stage_ms["gate_up"]
    # ---- aux-loss-free balancing step that follows routing in training: one
    # small kernel over the E counts (launch-latency bound); timed on its own.
    bias_scratch = inp["bias"].clone() if inp["bias"] is not None else torch.zeros(E, device=dev)
    ent = torch.empty(1, device=dev)
    # 100 calls captured in one CUDA graph, so the device time per call is
    # measured rather than the host's launch rate.
    for _ in range(3):
        B.moe_balance_update(cfg, counts, bias_scratch, 0.15, ent)
    torch.cuda.synchronize()
    bal_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(bal_graph):
        for _ in range(100):
            B.moe_balance_update(cfg, counts, bias_scratch, 0.15, ent)
    bal_graph.replay()
    torch.cuda.synchronize()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record(stream)
    bal_graph.replay()
    b1.record(stream)
    torch.cuda.synchronize()
    del bal_graph
    balance = {"us_per_call": b0.elapsed_time(b1) * 10.0, "entropy": ent.item(),
               "ln_E": math.log(E), "gamma": 0.15, "bound": "launch latency (E-element kernel)"}
    gelu = measure_gelu_experts(B, cfg, inp, counts.cpu(), stream, max(3, min(args.steps, 20)))
    work, touched = stage_work(cfg, counts.cpu(), B.moe_forward_gathers_rows(cfg, inp["x"]))
    gelu["expert_weight_frac_hbm"] = gelu["expert_weight_gbs"] / peaks["hbm"]
    bwd = measure_backward(B, cfg, inp, touched, stream, max(3, min(args.steps, 10)))
    bwd["frac_tensor"] = bwd["tflops"] / peaks["tensor_sustained"]
    bwd["frac_hbm"] = bwd["gbs"] / peaks["hbm"]
    dom = max(names, key=lambda n: stage_ms[n])
    wd = work[dom]
    t_dom = stage_ms[dom] / 1e3
    hbm_time = wd["bytes"] / (peaks["hbm"] * 1e9)
    tc_time = wd["flops"] / (peaks["tensor_sustained"] * 1e12)
    if tc_time > hbm_time:
        roof = {"bound": "tensor", "achieved": wd["flops"] / t_dom / 1e12, "peak": peaks["tensor_sustained"],
                "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": wd["bytes"] / t_dom / 1e9, "peak": peaks["hbm"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    # For context, against B200's nominal figures (HBM3e 7.7 TB/s HGX, dense bf16 2.25 PFLOP/s).
    roof["nominal_peak"] = 7700.0 if roof["bound"] == "hbm" else 2250.0
    roof["frac_nominal"] = roof["achieved"] / roof["nominal_peak"]
    roof["traffic"] = traffic_for(cfg.name, dom)
    roof.update({"kernel": dom, "peak_source": peaks["source"], "algorithmic_bytes": wd["bytes"],
                 "algorithmic_flops": wd["flops"], "kernel_ms": stage_ms[dom]})
    expert_ms = stage_ms["gate_up"] + stage_ms["down"]
    expert_flops = work["gate_up"]["flops"] + work["down"]["flops"]
    expert_bytes = work["gate_up"]["bytes"] + work["down"]["bytes"]

    # ---- end to end through the public call with host buffers ------------------
    # Every step copies its x from pinned host memory, runs moe_forward and copies
    # y back to pinned host memory. Copies run on their own streams with two
    # buffers, so step i's compute overlaps step i+1's upload and step i-1's
    # download, as a serving loop would.
    x_host = [inp["x"].cpu().pin_memory() for _ in range(2)]
    y_host = [torch.empty((T, d), dtype=cfg.torch_dtype).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(inp["x"]) for _ in range(2)]
    y_dev = [torch.empty_like(y) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=False)
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def e2e_run(n_steps, t_start, t_end):
        t_start.record(stream)
        s_in.wait_event(t_start)
        s_out.wait_event(t_start)
        for i in range(n_steps):
            b = i & 1
            if i >= 2:
                s_in.wait_event(comp_done[b])        # x_dev[b] no longer read
            with torch.cuda.stream(s_in):
                x_dev[b].copy_(x_host[b], non_blocking=True)
            in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            if i >= 2:
                stream.wait_event(out_done[b])       # y_dev[b] already downloaded
            B.moe_forward(cfg, x_dev[b], inp["w_router"], inp["bias"], inp["w1"], inp["w3"], inp["w2"],
                          inp["ws1"], inp["ws3"], inp["ws2"], y_dev[b], ws, stream)
            comp_done[b].record(stream)
            s_out.wait_event(comp_done[b])
            with torch.cuda.stream(s_out):
                y_host[b].copy_(y_dev[b], non_blocking=True)
            out_done[b].record(s_out)
        stream.wait_event(out_done[(n_steps - 1) & 1])
        if n_steps > 1:
            stream.wait_event(out_done[n_steps & 1])
        t_end.record(stream)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(3, e0, e1)
    torch.cuda.synchronize()
    barrier()
    e2e_run(args.steps, e0, e1)
    torch.cuda.synchronize()
    assert torch.equal(y_host[(args.steps - 1) & 1], y.cpu()), "end-to-end output differs"
    e2e_ms = reduce_max(e0.elapsed_time(e1) / args.steps, dev, world)
    barrier()

    # ---- CPU oracle baseline (rank 0, one GPU only) --------------------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n = min(CPU_SAMPLE_TOKENS.get(args.config, 16), T)
        dt, threads = oracle_sample_time(cfg, inp, n, seed=7)
        cpu = {"value": n / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} seeded tokens of {cfg.name}: fp64 routing over all {E} experts and the "
                         f"FFN of each selected and shared expert ({dt:.1f} s)"}

    sampler.stop()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if cfg.dtype == "bf16" else "f32", "data": "synthetic",
            "config": workload_config(cfg, world), "cuda_graph": graph is not None,
            "active_tflops": cfg.active_flops() * world / (ms_step / 1e3) / 1e12,
            "experts_touched": touched,
            "expert_gemm": {"ms": expert_ms, "tflops": expert_flops / (expert_ms / 1e3) / 1e12,
                            "gbs": expert_bytes / (expert_ms / 1e3) / 1e9,
                            "frac_tensor": expert_flops / (expert_ms / 1e3) / 1e12 / peaks["tensor_sustained"],
                            "frac_hbm": expert_bytes / (expert_ms / 1e3) / 1e9 / peaks["hbm"]},
            "stages_ms": stage_ms,
            "stages_ms_back_to_back": stage_iso,
            "balance_update": balance,
            "gelu_experts": gelu,
            "fused_permute_gather": fused,
            "backward": bwd,
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": whole_job_rate(T, world, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": T * d * cfg.elem_bytes, "d2h_bytes_per_step": T * d * cfg.elem_bytes,
                    "ms_per_step": e2e_ms},
            "workloads": extra,
            "gpu_launches": kernels_per_forward(B, cfg, inp["x"]) * args.steps,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if graph is not None:
        del graph
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
