#!/usr/bin/env python
"""Benchmark of the MixQ outlier-decomposed mixed-precision linear layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl mixq|reference]

One step is one pass of the whole hot path over one batch of every case of the
workload: the fused quantize/outlier-detection kernel, then the W8A8 and the
W4A8 mixed-precision GEMMs on the same quantized activations (two linear
layers sharing an input, one with 8-bit and one with 4-bit weights).  Weights
are prepacked once before timing (an offline step).  Every case has its own
weight copies, so a step touches more bytes than the 126 MB L2 and nothing is
served from L2 across steps.

The step is captured once in a CUDA graph (decode-sized kernels run for a few
microseconds, shorter than their host launch cost) and replayed; events around
the replays time the steps.  Copies of the graph with events at the phase
boundaries (quantize / W8A8 / W4A8), replayed right after, time each kernel
kind.  The end-to-end leg moves every step's inputs in from pinned host memory
and its outputs back, overlapping neighbouring steps' copies with the kernels.
Prints ONE JSON line on rank 0.

--impl reference times the CPU oracle (the plain C restatement of the layer)
on the host cores as the reference arm, on a bounded sample of the same
workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "mixed-precision GEMM TOPS and % of INT8 roofline (HBM GB/s at small M)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ workloads
def workload_cases(name: str, case_filter: str | None = None, modes: str | None = None):
    """(description, [(case, modes)]) -- each case runs quantize + one GEMM per mode.
    case_filter keeps the cases whose name contains it; modes overrides ("w8", "w4", "w8,w4")."""
    desc, cases = _workload_cases(name)
    if case_filter:
        cases = [(c, m) for c, m in cases if case_filter in c.name]
        desc += f" [only cases matching {case_filter!r}]"
    if modes:
        ms = tuple(x for x in modes.split(",") if x)
        cases = [(c, ms) for c, _ in cases]
        desc += f" [modes {','.join(ms)}]"
    if not cases:
        raise SystemExit("no case left after filtering")
    return desc, cases


def _workload_cases(name: str):
    if name == "llama7b-decode":
        return ("Llama-7B decode shapes, W8A8 and W4A8 on shared activations: M in {1,8,16,64} x "
                "(K,N) in {(4096,4096),(4096,11008),(11008,4096)}, 64 outlier channels x U[20,60]",
                [(c, ("w8", "w4")) for c in synth.decode("w8")])
    if name == "llama7b-prefill":
        return ("Llama-7B prefill shapes, W8A8 and W4A8: M in {512,2048,8192}, K=4096, N in "
                "{4096,11008}, outlier channels {0,32,128,256}",
                [(c, ("w8", "w4")) for c in synth.prefill("w8")])
    if name == "llama70b-b512":
        return ("Llama-70B shapes at batch 512, W8A8 and W4A8: (K,N) in {(8192,8192),(8192,28672),"
                "(28672,8192)}, 128 outlier channels unscaled (fast path) and x50",
                [(c, ("w8", "w4")) for c in synth.llama70b("w8")])
    if name == "tiny":
        return ("tiny W8A8+W4A8 layer: M=16, K=N=256, channels {3,77,130,201} x40",
                [(c, ("w8", "w4")) for c in synth.tiny()])
    raise SystemExit(f"unknown workload {name}")


def gemm_bytes(mode, M, N, K, k_out):
    """Algorithmic HBM bytes of one GEMM launch: weights (8-bit codes, or 4-bit codes plus one
    fp16 (s2, z2) pair per 128 weights), s_w, W_out, Xq, s_x, X_out, Y."""
    w = N * K if mode == "w8" else N * K // 2 + 4 * N * K // 128
    return w + 4 * N + 2 * N * k_out + M * K + 4 * M + 2 * M * k_out + 2 * M * N


def quant_bytes(M, K, k_out, norm=False):
    """Activation pass: read X, write Xq, X_out and s_x (plus the gain when the RMS
    normalisation is absorbed)."""
    kp = (k_out + 63) // 64 * 64
    return 2 * M * K + M * K + 2 * M * kp + 4 * M + (2 * K if norm else 0)


NORM_EPS = 1e-5


def gemm_ops(M, N, K, k_out, mixed):
    return 2 * M * N * K + (2 * M * N * k_out if mixed else 0)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def quantize_launches(M: int, K: int) -> int:
    """Kernels one mixq_quantize_act call launches: one cluster for decode-sized M
    (at most 16 CTAs of 1024 threads), else a reset pass and the main pass."""
    nvec = K // 8
    if 0 < M <= 64 and ((nvec <= 512 and (M + 1) // 2 <= 16) or (512 < nvec <= 2048 and M <= 16)):
        return 1
    return 2


def _code_only(text: str) -> str:
    """C/C++ source without its comments and blank lines (string literals kept)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"':  # string literal: copy through the closing quote
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            i = text.find("\n", i)
            i = n if i < 0 else i
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return "\n".join(ln.rstrip() for ln in "".join(out).splitlines() if ln.strip())


# The sources each measured kernel kind is compiled and configured from (its
# device code, the inline-PTX and tensor-map helpers, the shared constants, and
# the planner that picks its launch shape).  Committed ncu counters of a kind
# stay valid while these files' code is unchanged.
KERNEL_SOURCES = {
    "quantize": ("quantize.cu", "ptx.cuh", "internal.h"),
    "quantize_reset": ("quantize.cu", "ptx.cuh", "internal.h"),
    "gemm_w8": ("gemm.cu", "ptx.cuh", "tma_host.h", "internal.h"),
    "gemm_w4": ("gemm_w4ts.cu", "gemm.cu", "ptx.cuh", "tma_host.h", "internal.h"),
    "prepack": ("prepack.cu", "ptx.cuh", "internal.h"),
}


def kernel_source_hash(kind: str | None = None) -> str:
    """Hash of the code (comments stripped) of the kernel source files: those of one
    kernel kind, or every file under csrc/ when kind is None."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mixed_precision_quantized_mixq_b200", "csrc")
    if kind is None:
        files = sorted(f for f in os.listdir(csrc) if f.endswith((".cu", ".cuh", ".h")))
    else:
        files = sorted(KERNEL_SOURCES[kind])
    for f in files:
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(f.encode() + b"\0" + _code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def load_traffic(kernel_kind: str, workload: str, path: str | None = None):
    """Per-launch DRAM bytes of a kernel from the committed ncu summary, or None if the
    summary is missing or was taken on different sources of that kernel."""
    p = path or os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        if d["source_hashes"][kernel_kind] != kernel_source_hash(kernel_kind):
            return None
        return d["workloads"][workload][kernel_kind]["bytes_per_launch"]
    except Exception:
        return None


# ------------------------------------------------------------ clock sampling
class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.proc = None
        self.t0 = self.t1 = None
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if gpu_id:
            cmd += ["-i", gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None

    def mark(self, start: bool):
        if start:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
            except Exception:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        lo = (self.t0 or 0) - 1.0
        hi = (self.t1 or 1e18) + 1.0
        inside = [r for r in rows if lo <= r[0] <= hi] or rows
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in inside for n, v in zip(names, r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "samples": len(inside)}


# ------------------------------------------------------- multi-rank helpers
def rank_activations(case, rank: int):
    """Activations of one case for one rank: rank 0 uses the workload's own
    seeded tensor, rank r > 0 an independent draw (seed offset 1000 r) of the
    same distribution -- each rank processes its own batch (weak scaling)."""
    idx = case.channels()
    seed = synth.SEED_X + 1000 * rank
    if case.scaled and case.k_out:
        f = case.factor if case.factor is not None else synth.channel_factors(case.k_out)
        return synth.activations(case.M, case.K, idx, f, seed=seed), idx
    return synth.activations(case.M, case.K, seed=seed), idx


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Largest value across ranks (a no-op for one rank)."""
    if world <= 1:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- GPU arm
def run_gpu(args, rank, world):
    import torch

    import mixed_precision_quantized_mixq_b200 as mq

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    desc, cases = workload_cases(args.workload, args.case, args.modes)
    T = synth.THRESHOLD

    # ---- inputs and offline prepack (untimed); inputs differ per rank (weak scaling)
    weights_host = {}
    layers = []
    for ci, (case, modes) in enumerate(cases):
        X, idx = rank_activations(case, rank)
        key = (case.N, case.K)
        if key not in weights_host:
            weights_host[key] = synth.weights(case.N, case.K)
        Wd = torch.from_numpy(weights_host[key]).to(dev)
        idxd = torch.from_numpy(idx).to(dev)
        packed = {m: mq.prepack(Wd, idxd, mq.MIXQ_W8 if m == "w8" else mq.MIXQ_W4G128)
                  for m in modes}
        del Wd
        gamma = torch.from_numpy(synth.gains(case.K)).to(dev) if args.norm else None
        layers.append(dict(case=case, modes=modes, Xh=X, idx=idxd, packed=packed, gamma=gamma))
    weights_host.clear()
    # All activations of a step live in one device buffer and all outputs in
    # another (per-case views), so the end-to-end leg moves each with a single
    # host<->device copy.
    x_sizes = [L["case"].M * L["case"].K for L in layers]
    y_sizes = [L["case"].M * L["case"].N * len(L["modes"]) for L in layers]
    X_all = torch.empty(sum(x_sizes), dtype=torch.float16, device=dev)
    Y_all = torch.empty(sum(y_sizes), dtype=torch.float16, device=dev)

    def bind(Xb, Yb):
        """Per-case views (X, Y per mode) of one packed activation/output buffer pair."""
        views, xo, yo = [], 0, 0
        for L, xs, ys in zip(layers, x_sizes, y_sizes):
            c = L["case"]
            V = {"X": Xb[xo:xo + xs].view(c.M, c.K), "Y": {}}
            for mi, m in enumerate(L["modes"]):
                V["Y"][m] = Yb[yo + mi * c.M * c.N: yo + (mi + 1) * c.M * c.N].view(c.M, c.N)
            views.append(V)
            xo += xs
            yo += ys
        return views

    def act_pass(L, V, out=None):
        if args.norm:
            return mq.rmsnorm_quantize_act(V["X"], L["gamma"], NORM_EPS, L["idx"], T, out=out,
                                           status=status)
        return mq.quantize_act(V["X"], L["idx"], T, out=out, status=status)

    status = torch.zeros(1, dtype=torch.int32, device=dev)
    views0 = bind(X_all, Y_all)
    for L, V in zip(layers, views0):
        V["X"].copy_(torch.from_numpy(L.pop("Xh")))
        V["q"] = act_pass(L, V)
    torch.cuda.synchronize()

    modes_all = []
    for L in layers:
        for m in L["modes"]:
            if m not in modes_all:
                modes_all.append(m)

    def step(events=None, views=None):
        # Phase order: every case's quantize, then every case's W8A8 GEMM, then
        # every W4A8 GEMM.  Timing events sit only at the phase boundaries, so
        # consecutive kernels keep overlapping (programmatic dependent launch).
        views = views0 if views is None else views
        if events is not None:
            events[0].record()
        for L, V in zip(layers, views):
            act_pass(L, V, out=V["q"])
        if events is not None:
            events[1].record()
        for mi, m in enumerate(modes_all):
            for L, V in zip(layers, views):
                if m in L["modes"]:
                    mq.gemm(V["q"], L["packed"][m], Y=V["Y"][m], status=status)
            if events is not None:
                events[2 + mi].record()

    # eager warm-up (initializes kernels and attributes before capture), then check status
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    mq.check_status(status)
    mixed = [int(V["q"].flags[0].item()) > 0 for V in views0]

    # ---- the step as one CUDA graph (the timed region of the whole-step value), and
    # up to 32 copies with timing events at the phase boundaries, replayed once each
    # right after it: their events give the per-kernel-kind durations.  (Event nodes
    # inside a graph cost the chained kernels some of their overlap, about 5 % of a
    # decode step, so they stay out of the value's timed region.)
    side = torch.cuda.Stream(device=dev)
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=side):
        step()
    n_graphs = min(args.steps, 32)
    graphs, ev_sets = [], []
    for g_i in range(n_graphs):
        evs = [torch.cuda.Event(enable_timing=True, external=True)
               for _ in range(2 + len(modes_all))]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            step(evs)
        graphs.append(g)
        ev_sets.append(evs)
    torch.cuda.synchronize()

    for i in range(args.warmup):
        g_step.replay()
    torch.cuda.synchronize()

    gpu_id = None
    try:
        gpu_id = str(torch.cuda.get_device_properties(dev).uuid)
        gpu_id = gpu_id if gpu_id.startswith("GPU-") else "GPU-" + gpu_id
    except Exception:
        gpu_id = None
    sampler = ClockSampler(gpu_id)
    time.sleep(0.3)

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.mark(True)
    start.record()
    for i in range(args.steps):
        g_step.replay()
    end.record()
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    sampler.mark(False)
    if world > 1:
        torch.distributed.barrier()
    total_ms = start.elapsed_time(end)
    clocks = sampler.stop()
    mq.check_status(status)

    total_ms = max_over_ranks(total_ms, world, dev)

    # ---- per-kernel durations from the in-graph phase events
    kinds = {"quantize": [0.0, 0.0, 0], "gemm_w8": [0.0, 0.0, 0], "gemm_w4": [0.0, 0.0, 0]}
    for evs in ev_sets:
        kinds["quantize"][0] += evs[0].elapsed_time(evs[1])
        for mi, m in enumerate(modes_all):
            kinds["gemm_" + m][0] += evs[1 + mi].elapsed_time(evs[2 + mi])
        for L in layers:
            c = L["case"]
            kinds["quantize"][1] += quant_bytes(c.M, c.K, c.k_out, args.norm)
            kinds["quantize"][2] += 1
            for m in L["modes"]:
                kinds["gemm_" + m][1] += gemm_bytes(m, c.M, c.N, c.K, c.k_out)
                kinds["gemm_" + m][2] += 1
    ops_step = sum(gemm_ops(L["case"].M, L["case"].N, L["case"].K, L["case"].k_out, mixed[i])
                   for i, L in enumerate(layers) for _ in L["modes"])
    kind_ops = {"gemm_w8": 0.0, "gemm_w4": 0.0, "quantize": 0.0}
    for i, L in enumerate(layers):
        c = L["case"]
        for m in L["modes"]:
            kind_ops["gemm_" + m] += gemm_ops(c.M, c.N, c.K, c.k_out, mixed[i]) * n_graphs

    ms_per_step = total_ms / args.steps
    value = ops_step * world / (ms_per_step * 1e-3) / 1e12  # TOPS, all ranks

    peaks, peak_src = load_peaks()
    dom = max(kinds, key=lambda k: kinds[k][0])
    t_ms, bytes_tot, launches = kinds[dom]
    gbs = bytes_tot / (t_ms * 1e-3) / 1e9
    tops = kind_ops[dom] / (t_ms * 1e-3) / 1e12
    i8_peak = 2.0 * (peaks["bf16_tflops_sustained"] if total_ms > 1000 else peaks["bf16_tflops"])
    t_c = kind_ops[dom] / (i8_peak * 1e12)
    t_m = bytes_tot / (peaks["hbm_gbs"] * 1e9)
    traffic = load_traffic(dom, args.workload)
    if t_m >= t_c:
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": traffic}
    else:
        roof = {"bound": "tensor", "achieved": round(tops, 1), "peak": round(i8_peak, 1),
                "unit": "TFLOP/s", "frac": round(tops / i8_peak, 4), "traffic": traffic}
    roof.update({"kernel": dom, "launches_timed": launches,
                 "avg_launch_us": round(1e3 * t_ms / launches, 3),
                 "algorithmic_bytes_per_step": int(bytes_tot / n_graphs),
                 "peak_source": f"{peak_src} MEASURED_PEAKS.json" if peak_src == "measured" else
                 "fallback (6.65 TB/s, 1.59 PFLOP/s bf16)",
                 "int8_peak_rule": "2 x measured bf16 TFLOP/s (nominal int8:bf16 ratio)",
                 "share_of_step": {k: round(v[0] / max(1e-9, sum(x[0] for x in kinds.values())), 4)
                                   for k, v in kinds.items()},
                 # every kernel kind against the HBM copy rate (algorithmic bytes / time)
                 "per_kind": {k: {"avg_launch_us": round(1e3 * v[0] / max(1, v[2]), 3),
                                  "GB/s": round(v[1] / max(1e-12, v[0] * 1e-3) / 1e9, 1),
                                  "frac_hbm": round(v[1] / max(1e-12, v[0] * 1e-3) / 1e9
                                                    / peaks["hbm_gbs"], 4)}
                              for k, v in kinds.items()}})

    # ---- end to end: host X in pinned memory -> device -> layer -> Y back to pinned host.
    # Every step copies its inputs in and its outputs out; two device buffer sets
    # let step i+1's input copy and step i-1's output copy run beside step i's
    # kernels (three streams, ordered by events).
    host_X = X_all.cpu().pin_memory()
    host_Y = torch.empty(Y_all.shape, dtype=torch.float16).pin_memory()
    h2d = host_X.numel() * 2
    d2h = host_Y.numel() * 2
    X_all1, Y_all1 = torch.empty_like(X_all), torch.empty_like(Y_all)
    views1 = bind(X_all1, Y_all1)
    X_all1.copy_(X_all)
    for L, V in zip(layers, views1):
        V["q"] = act_pass(L, V)
    torch.cuda.synchronize()
    bufX, bufY = (X_all, X_all1), (Y_all, Y_all1)
    ge = []
    for views in (views0, views1):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            step(views=views)
        ge.append(g)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run_e2e(n, start_ev=None, end_ev=None):
        if start_ev is not None:
            start_ev.record(s_in)
        with torch.cuda.stream(s_in):
            bufX[0].copy_(host_X, non_blocking=True)
            ev_in[0].record(s_in)
        for i in range(n):
            b = i % 2
            if i + 1 < n:  # next step's input, once step i-1 is done reading that buffer
                nb = (i + 1) % 2
                s_in.wait_event(ev_comp[nb])
                with torch.cuda.stream(s_in):
                    bufX[nb].copy_(host_X, non_blocking=True)
                    ev_in[nb].record(s_in)
            side.wait_event(ev_in[b])
            side.wait_event(ev_out[b])  # step i-2's output copy is out of Y[b]
            with torch.cuda.stream(side):
                ge[b].replay()
                ev_comp[b].record(side)
            s_out.wait_event(ev_comp[b])
            with torch.cuda.stream(s_out):
                host_Y.copy_(bufY[b], non_blocking=True)
                ev_out[b].record(s_out)
        if end_ev is not None:
            end_ev.record(s_out)

    run_e2e(max(3, args.warmup))
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run_e2e(args.steps, s2, e2)
    torch.cuda.synchronize()
    e2e_ms = s2.elapsed_time(e2)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    mq.check_status(status)
    e2e = {"value": round(ops_step * world / (e2e_ms / args.steps * 1e-3) / 1e12, 4),
           "unit": "TOPS", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "ms_per_step": round(e2e_ms / args.steps, 5),
           "how": "per step: one pinned-host -> device copy of every case's X, quantize + both "
                  "GEMMs (CUDA graph), one device -> pinned-host copy of every Y; copies of "
                  "neighbouring steps overlap the kernels (two device buffer sets, three streams)"}

    launches_per_step = sum(quantize_launches(L["case"].M, L["case"].K) + len(L["modes"])
                            for L in layers)
    touched = sum(L["packed"][m].Wq.numel() * L["packed"][m].Wq.element_size()
                  for L in layers for m in L["modes"])
    result = {
        "metric": METRIC, "value": round(value, 4), "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8 (int8 x int8 -> int32 tensor cores) + fp16 outlier slice (fp32 accumulate)",
        "data": "synthetic (seeded normals; random-init weights of the Llama shapes)",
        "config": {"workload": args.workload, "description": desc, "cases": len(layers),
                   "activation_pass": ("RMS normalisation (seeded gain ~N(1,0.1), eps 1e-5) "
                                       "absorbed into the quantize kernel" if args.norm else
                                       "quantize (amax, threshold, gather, int8)"),
                   "mixed_tokens_per_case": [int(V["q"].flags[0].item()) for V in views0],
                   "l2": f"inputs larger than L2: {touched / 1e6:.0f} MB of distinct weights per "
                         "step (126 MB L2), each case reads its own copy",
                   "launch": "one CUDA graph per step (captured once, replayed); kernels chained "
                             "with programmatic dependent launch; step order: all quantize, "
                             "all W8A8 GEMMs, all W4A8 GEMMs; per-kernel-kind times from "
                             "graph copies with events at the phase boundaries, replayed after "
                             "the timed steps",
                   "parallelism": f"dp{world} (independent batches per GPU, no collective)"},
        "roofline": roof,
        "e2e": e2e,
        "clocks": clocks,
        "gpu_launches": launches_per_step * args.steps,
    }
    return result


# -------------------------------------------------------------- CPU oracle
def oracle_prepare(cases, norm=False):
    """Oracle inputs for every case: activations, and weights prepacked by the oracle
    (prepack is offline and not timed).  Weights are drawn once per shape.  With norm
    each item carries the RMS-normalisation gain."""
    import oracle
    wraw, wcache, prepared = {}, {}, []
    for case, modes in cases:
        idx = case.channels()
        if case.scaled and case.k_out:
            f = case.factor if case.factor is not None else synth.channel_factors(case.k_out)
            X = synth.activations(case.M, case.K, idx, f)
        else:
            X = synth.activations(case.M, case.K)
        key = (case.N, case.K, case.k_out)
        if key not in wcache:
            if (case.N, case.K) not in wraw:
                wraw[(case.N, case.K)] = synth.weights(case.N, case.K)
            Wq8, s_w, W_out = oracle.prepack_w8(wraw[(case.N, case.K)], idx)
            _, _, _, w8eff = oracle.prepack_w4(Wq8)
            wcache[key] = {"w8": (Wq8, s_w, W_out), "w4": (w8eff, s_w, W_out)}
        prepared.append((case, modes, X, idx, wcache[key], synth.gains(case.K) if norm else None))
    return prepared


def oracle_unit(item, m, ns):
    """The layer for token m of one case at output channels ns (all modes): quantize the
    token, then the mixed-precision product at each sampled output.  Returns GEMM ops."""
    import oracle
    case, modes, X, idx, w, gamma = item
    x = X[m:m + 1] if gamma is None else oracle.rmsnorm(X[m:m + 1], gamma, NORM_EPS)
    Xq, s_x, X_out, _, flags = oracle.quantize_act(x, idx, case.threshold)
    ms = np.zeros(len(ns), np.int32)
    ops = 0
    for mode in modes:
        Wq, s_w, W_out = w[mode]
        xo = X_out if X_out.shape[1] else None
        wo = W_out if W_out.shape[1] else None
        oracle.linear_points(Xq, s_x, xo, Wq, s_w, wo, ms, ns)
        ops += len(ns) * (2 * case.K + (2 * case.k_out if flags[0] > 0 else 0))
    return ops


class OracleSampler:
    """Bounded samples of the workload for the CPU oracle: unit i is token (i // cases)
    of case (i % cases) at `points` output channels drawn from a seeded stream."""

    def __init__(self, prepared, points):
        self.prepared, self.points, self.i = prepared, points, 0
        self.rng = np.random.default_rng(7)

    def run(self, units):
        ops = 0
        for _ in range(units):
            item = self.prepared[self.i % len(self.prepared)]
            m = (self.i // len(self.prepared)) % item[0].M
            ns = self.rng.integers(0, item[0].N, self.points).astype(np.int32)
            ops += oracle_unit(item, m, ns)
            self.i += 1
        return ops


def calibrate(sampler, target_s):
    """Units per step so that one step takes about target_s."""
    t0 = time.perf_counter()
    sampler.run(len(sampler.prepared))
    per_unit = (time.perf_counter() - t0) / len(sampler.prepared)
    return max(1, int(target_s / max(per_unit, 1e-6)))


def cpu_cores(points):
    n = os.cpu_count() or 1
    env = os.environ.get("OMP_NUM_THREADS")
    if env and env.isdigit():
        n = int(env)
    return min(n, points)


def run_cpu_baseline(args, budget_s=15.0):
    _, cases = workload_cases(args.workload, args.case, args.modes)
    points = 2048
    sampler = OracleSampler(oracle_prepare(cases, args.norm), points)
    units = calibrate(sampler, budget_s)
    t0 = time.perf_counter()
    ops = sampler.run(units)
    dt = time.perf_counter() - t0
    return {"value": round(ops / dt / 1e12, 6), "unit": "TOPS", "cores": cpu_cores(points),
            "kind": "oracle",
            "sample": f"{units} units of (one token of one case, quantize + W8A8 + W4A8 at "
                      f"{points} sampled output channels), cycling over the "
                      f"{len(sampler.prepared)} cases; plain C, OpenMP over outputs; {dt:.1f} s"}


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle on the host cores, same metric and workload; each step
    is a bounded sample sized so the whole run takes about a minute."""
    if rank != 0:
        return None
    desc, cases = workload_cases(args.workload, args.case, args.modes)
    points = 2048
    sampler = OracleSampler(oracle_prepare(cases, args.norm), points)
    step_s = min(0.5, 60.0 / (args.steps + args.warmup))
    units = calibrate(sampler, step_s)
    sampler.run(units * args.warmup)
    t0 = time.perf_counter()
    ops = sampler.run(units * args.steps)
    dt = time.perf_counter() - t0
    value = ops / dt / 1e12
    sample = (f"per step: {units} units of (one token of one case, quantize + W8A8 + W4A8 at "
              f"{points} sampled output channels), cycling over the {len(cases)} cases")
    return {"metric": METRIC, "value": round(value, 6), "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8 codes, int64/fp64 accumulate",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": args.workload, "description": desc},
            "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": cpu_cores(points),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", default="llama7b-decode",
                    choices=["llama7b-decode", "llama7b-prefill", "llama70b-b512", "tiny"])
    ap.add_argument("--impl", default="mixq", choices=["mixq", "reference"])
    ap.add_argument("--case", default=None, help="keep only cases whose name contains this")
    ap.add_argument("--modes", default=None, help="weight formats to run: w8, w4 or w8,w4")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--norm", action="store_true",
                    help="absorb an RMS normalisation of each token (seeded gain ~N(1,0.1), "
                         "eps 1e-5) into the activation pass")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0

    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res = run_gpu(args, rank, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = run_cpu_baseline(args)
    elif rank == 0:
        res["cpu_baseline"] = None
    if world > 1:
        import torch
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
