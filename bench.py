#!/usr/bin/env python
"""Benchmark of the MixQ outlier-decomposed mixed-precision linear layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--decode-workload NAME | --no-decode] [--modes w8,w4,w4b]
                    [--impl mixq|reference]

One step is one pass of the whole hot path over one batch of every case of the
workload: the fused quantize/outlier-detection kernel, then one mixed-precision
GEMM per weight format on the same quantized activations (linear layers that
share an input: W8A8, W4A8 with progressive 4-bit weights, and optionally W4A8
with fp16 group scales).  Weights are prepacked once before timing (an offline
step).  Every case has its own weight copies, so a step touches more bytes
than the 126 MB L2 and nothing is served from L2 across steps.

The headline line measures the large-M workload (default: the Llama-7B prefill
sweep, M up to 8192), whose GEMMs are bound by the INT8 tensor pipe; its
roofline peak is the INT8 MMA rate of this GPU, measured in the same run by the
library's own tcgen05 kind::i8 rate loop for as long as the timed region.  A
`decode` sub-record measures the small-M workload (default: the Llama-7B decode
sweep), whose GEMMs are bound by HBM, with per-kernel-kind HBM fractions.

Each step is captured once in a CUDA graph (decode-sized kernels run for a few
microseconds, shorter than their host launch cost) and replayed; events around
the replays time the steps.  Copies of the graph with events at the phase
boundaries (quantize / each GEMM kind), replayed right after, time each kernel
kind.  The end-to-end leg moves every step's inputs in from pinned host memory
and its outputs back, overlapping neighbouring steps' copies with the kernels.
Prints ONE JSON line on rank 0.  `--gpus N` starts one process per GPU (torch
distributed, NCCL) when it is not already running under a launcher.

--impl reference times the CPU oracle (the plain C restatement of the layer)
on the host cores as the reference arm, on a bounded sample of the same
workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import socket
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
WORKLOADS = ["llama7b-prefill", "llama7b-decode", "llama70b-b512", "tiny"]
DEFAULT_MODES = {"llama7b-prefill": "w8,w4", "llama70b-b512": "w8,w4", "tiny": "w8,w4",
                 "llama7b-decode": "w8,w4,w4b"}
MODE_NAMES = {"w8": "W8A8", "w4": "W4A8 (progressive 4-bit, integer group scale)",
              "w4b": "W4A8 (4-bit, fp16 group scale and integer zero)"}


# ------------------------------------------------------------------ workloads
def workload_cases(name: str, case_filter: str | None = None, modes: str | None = None):
    """(description, [(case, modes)]) -- each case runs quantize + one GEMM per mode.
    case_filter keeps the cases whose name contains it; modes overrides the workload's
    default weight formats ("w8", "w4", "w4b", comma separated)."""
    desc, cases = _workload_cases(name)
    ms = tuple(x for x in (modes or DEFAULT_MODES[name]).split(",") if x)
    for m in ms:
        if m not in MODE_NAMES:
            raise SystemExit(f"unknown weight format {m}")
    cases = [(c, ms) for c in cases]
    desc += "; weight formats: " + ", ".join(MODE_NAMES[m] for m in ms)
    if case_filter:
        cases = [(c, m) for c, m in cases if case_filter in c.name]
        desc += f" [only cases matching {case_filter!r}]"
    if not cases:
        raise SystemExit("no case left after filtering")
    return desc, cases


def _workload_cases(name: str):
    if name == "llama7b-decode":
        return ("Llama-7B decode shapes: M in {1,8,16,64} x (K,N) in {(4096,4096),(4096,11008),"
                "(11008,4096)}, 64 outlier channels x U[20,60]", synth.decode("w8"))
    if name == "llama7b-prefill":
        return ("Llama-7B prefill shapes: M in {512,2048,8192}, K=4096, N in {4096,11008}, "
                "outlier channels {0,32,128,256} x U[20,60]", synth.prefill("w8"))
    if name == "llama70b-b512":
        return ("Llama-70B shapes at batch 512: (K,N) in {(8192,8192),(8192,28672),(28672,8192)}, "
                "128 outlier channels unscaled (fast path) and x50", synth.llama70b("w8"))
    if name == "tiny":
        return ("tiny layer: M=16, K=N=256, channels {3,77,130,201} x40", synth.tiny())
    raise SystemExit(f"unknown workload {name}")


def gemm_bytes(mode, M, N, K, k_out):
    """Algorithmic HBM bytes of one GEMM launch: weights (8-bit codes, or 4-bit codes plus one
    fp16 pair per 128 weights), s_w (not in the fp16-scale format), W_out, Xq, s_x, X_out, Y."""
    if mode == "w8":
        w = N * K + 4 * N
    elif mode == "w4":
        w = N * K // 2 + 4 * N * K // 128 + 4 * N
    else:
        w = N * K // 2 + 4 * N * K // 128
    return w + 2 * N * k_out + M * K + 4 * M + 2 * M * k_out + 2 * M * N


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
    one_cluster = (nvec <= 512 and (M + 3) // 4 <= 16) or \
        (512 < nvec <= 2048 and M <= 16) or (512 < nvec <= 1536 and (M + 1) // 2 <= 16)
    return 1 if 0 < M <= 64 and one_cluster else 2


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
    "gemm_w8": ("gemm.cu", "gemm_pair.cu", "ptx.cuh", "tma_host.h", "internal.h"),
    "gemm_w4": ("gemm_w4ts.cu", "gemm_pair_w4.cu", "gemm.cu", "ptx.cuh", "tma_host.h",
                "internal.h"),
    "gemm_w4b": ("gemm_w4b.cu", "gemm_w4b.h", "ptx.cuh", "tma_host.h", "internal.h"),
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
    """nvidia-smi sampling in the background; named windows are summarised at stop()."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.proc = None
        self.windows = {}
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if gpu_id:
            cmd += ["-i", gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None

    def mark(self, name: str, start: bool):
        w = self.windows.setdefault(name, [None, None])
        w[0 if start else 1] = time.time()

    def stop(self):
        """{window: {"sm_mhz": median, "sm_max_mhz", "reasons", "samples"}}."""
        if self.proc is None:
            return {n: {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
                    for n in self.windows}
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
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        res = {}
        for n, (t0, t1) in self.windows.items():
            if not rows:
                res[n] = {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
                continue
            lo, hi = (t0 or 0) - 1.0, (t1 or 1e18) + 1.0
            inside = [r for r in rows if lo <= r[0] <= hi] or rows
            reasons = sorted({nm for r in inside for nm, v in zip(names, r[3])
                              if v.lower() == "active"})
            res[n] = {"sm_mhz": statistics.median(r[1] for r in inside),
                      "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                      "samples": len(inside)}
        return res


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


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def launch_ranks(gpus: int, argv: list[str]) -> int:
    """Run this script as `gpus` processes, one per GPU, under torch's launcher
    (rendezvous on 127.0.0.1); returns the launcher's exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={gpus}", "--master-addr", "127.0.0.1",
           "--master-port", str(_free_port()), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


# ------------------------------------------------------- tensor-core peak
MMA_I8, MMA_F16 = 0, 1


def measure_mma_rate(mq, torch, dev, kind: int, seconds: float, status):
    """Rate (TOP/s) of the library's tcgen05.mma rate loop, run back to back for about
    `seconds`: {"median", "max", "launches", "seconds"}.  Launches of ~2 ms each."""
    s = torch.cuda.current_stream(dev)
    iters = 1024
    ops = mq.mixq_debug_mma_rate(kind, iters, status)  # also the first (warming) launch
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    mq.mixq_debug_mma_rate(kind, iters, status)
    e1.record(s)
    torch.cuda.synchronize(dev)
    per_iter_ms = max(1e-6, e0.elapsed_time(e1) / iters)
    iters = int(min(1 << 20, max(64, 2.0 / per_iter_ms)))
    n = int(max(3, min(2000, seconds * 1e3 / max(1e-3, per_iter_ms * iters))))
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
    evs[0].record(s)
    for i in range(n):
        ops = mq.mixq_debug_mma_rate(kind, iters, status)
        evs[i + 1].record(s)
    torch.cuda.synchronize(dev)
    rates = [ops / (evs[i].elapsed_time(evs[i + 1]) * 1e-3) / 1e12 for i in range(n)]
    return {"median": statistics.median(rates), "max": max(rates), "launches": n,
            "seconds": round(evs[0].elapsed_time(evs[n]) * 1e-3, 3)}


# ----------------------------------------------------------------- GPU arm
def measure_workload(mq, torch, dev, rank, world, workload, modes, steps, warmup, norm, sampler,
                     window, before_timed=None, want_e2e=True, case_filter=None):
    """Time one workload: whole-step value, per-kernel-kind durations, end to end.
    Returns a dict of raw measurements (see build_record)."""
    desc, cases = workload_cases(workload, case_filter, modes)
    T = synth.THRESHOLD
    fmt = {"w8": mq.MIXQ_W8, "w4": mq.MIXQ_W4G128, "w4b": mq.MIXQ_W4G128_F16S}

    # ---- inputs and offline prepack (untimed); inputs differ per rank (weak scaling)
    weights_host = {}
    layers = []
    for case, ms in cases:
        X, idx = rank_activations(case, rank)
        key = (case.N, case.K)
        if key not in weights_host:
            weights_host[key] = synth.weights(case.N, case.K)
        Wd = torch.from_numpy(weights_host[key]).to(dev)
        idxd = torch.from_numpy(idx).to(dev)
        packed = {m: mq.prepack(Wd, idxd, fmt[m]) for m in ms}
        del Wd
        gamma = torch.from_numpy(synth.gains(case.K)).to(dev) if norm else None
        layers.append(dict(case=case, modes=ms, Xh=X, idx=idxd, packed=packed, gamma=gamma))
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

    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def act_pass(L, V, out=None):
        if norm:
            return mq.rmsnorm_quantize_act(V["X"], L["gamma"], NORM_EPS, L["idx"], T, out=out,
                                           status=status)
        return mq.quantize_act(V["X"], L["idx"], T, out=out, status=status)

    views0 = bind(X_all, Y_all)
    for L, V in zip(layers, views0):
        V["X"].copy_(torch.from_numpy(L.pop("Xh")))
        V["q"] = act_pass(L, V)
    torch.cuda.synchronize(dev)

    modes_all = []
    for L in layers:
        for m in L["modes"]:
            if m not in modes_all:
                modes_all.append(m)

    def step(events=None, views=None):
        # Phase order: every case's quantize, then every case's GEMM of the first
        # weight format, then the next format.  Timing events sit only at the phase
        # boundaries, so consecutive kernels keep overlapping (programmatic
        # dependent launch).
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
    torch.cuda.synchronize(dev)
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
    n_graphs = min(steps, 32)
    graphs, ev_sets = [], []
    for _ in range(n_graphs):
        evs = [torch.cuda.Event(enable_timing=True, external=True)
               for _ in range(2 + len(modes_all))]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            step(evs)
        graphs.append(g)
        ev_sets.append(evs)
    torch.cuda.synchronize(dev)

    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0.record()
    for _ in range(warmup):
        g_step.replay()
    w1.record()
    torch.cuda.synchronize(dev)
    est_ms = w0.elapsed_time(w1) / max(1, warmup)
    extra = before_timed(est_ms * steps) if before_timed is not None else None

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.mark(window, True)
    start.record()
    for _ in range(steps):
        g_step.replay()
    end.record()
    torch.cuda.synchronize(dev)
    sampler.mark(window, False)
    for g in graphs:
        g.replay()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    total_ms = max_over_ranks(start.elapsed_time(end), world, dev)
    mq.check_status(status)

    # ---- per-kernel durations from the in-graph phase events
    kinds = {"quantize": [0.0, 0.0, 0, 0.0]}
    for m in modes_all:
        kinds["gemm_" + m] = [0.0, 0.0, 0, 0.0]  # ms, bytes, launches, ops
    for evs in ev_sets:
        kinds["quantize"][0] += evs[0].elapsed_time(evs[1])
        for mi, m in enumerate(modes_all):
            kinds["gemm_" + m][0] += evs[1 + mi].elapsed_time(evs[2 + mi])
        for i, L in enumerate(layers):
            c = L["case"]
            kinds["quantize"][1] += quant_bytes(c.M, c.K, c.k_out, norm)
            kinds["quantize"][2] += 1
            for m in L["modes"]:
                k = kinds["gemm_" + m]
                k[1] += gemm_bytes(m, c.M, c.N, c.K, c.k_out)
                k[2] += 1
                k[3] += gemm_ops(c.M, c.N, c.K, c.k_out, mixed[i])
    ops_step = sum(gemm_ops(L["case"].M, L["case"].N, L["case"].K, L["case"].k_out, mixed[i])
                   for i, L in enumerate(layers) for _ in L["modes"])
    launches_per_step = sum(quantize_launches(L["case"].M, L["case"].K) + len(L["modes"])
                            for L in layers)
    touched = sum(L["packed"][m].Wq.numel() * L["packed"][m].Wq.element_size()
                  for L in layers for m in L["modes"])
    res = dict(workload=workload, desc=desc, cases=len(layers), steps=steps, warmup=warmup,
               total_ms=total_ms, ops_step=ops_step, kinds=kinds, n_graphs=n_graphs,
               launches_per_step=launches_per_step, touched=touched, modes=modes_all,
               mixed_tokens=[int(V["q"].flags[0].item()) for V in views0], extra=extra)
    del graphs, ev_sets
    if not want_e2e:
        return res

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
    torch.cuda.synchronize(dev)
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

    run_e2e(max(3, warmup))
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run_e2e(steps, s2, e2)
    torch.cuda.synchronize(dev)
    res["e2e_ms"] = max_over_ranks(s2.elapsed_time(e2), world, dev)
    res["h2d"], res["d2h"] = h2d, d2h
    mq.check_status(status)
    del ge
    return res


def build_record(r, world, peaks, peak_src, i8_peak):
    """The JSON fields of one measured workload: value, roofline of the dominant kernel
    kind (and per kind), e2e.  i8_peak = (TOP/s, rule text) for tensor-bound kernels."""
    steps = r["steps"]
    ms_per_step = r["total_ms"] / steps
    value = r["ops_step"] * world / (ms_per_step * 1e-3) / 1e12  # TOPS, all ranks
    kinds, n_graphs = r["kinds"], r["n_graphs"]
    i8, i8_rule = i8_peak
    i8_2bf16 = 2.0 * (peaks["bf16_tflops_sustained"] if r["total_ms"] > 1000
                      else peaks["bf16_tflops"])
    dom = max(kinds, key=lambda k: kinds[k][0])
    t_ms, bytes_tot, launches, ops_tot = kinds[dom]
    gbs = bytes_tot / (t_ms * 1e-3) / 1e9
    tops = ops_tot / (t_ms * 1e-3) / 1e12
    t_c = ops_tot / (i8 * 1e12) if ops_tot else 0.0
    t_m = bytes_tot / (peaks["hbm_gbs"] * 1e9)
    traffic = load_traffic(dom, r["workload"])
    if t_m >= t_c:
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": traffic,
                "peak_source": ("measured MEASURED_PEAKS.json hbm_gbs" if peak_src == "measured"
                                else "fallback (6.65 TB/s)")}
    else:
        roof = {"bound": "tensor", "achieved": round(tops, 1), "peak": round(i8, 1),
                "unit": "TFLOP/s", "frac": round(tops / i8, 4), "traffic": traffic,
                "peak_source": i8_rule,
                "frac_vs_2x_bf16": round(tops / i8_2bf16, 4),
                "peak_2x_bf16": round(i8_2bf16, 1)}
    roof.update({
        "kernel": dom, "launches_timed": launches,
        "avg_launch_us": round(1e3 * t_ms / launches, 3),
        "algorithmic_bytes_per_step": int(bytes_tot / n_graphs),
        "algorithmic_ops_per_step": int(ops_tot / n_graphs),
        "int8_peak_rule": i8_rule,
        "share_of_step": {k: round(v[0] / max(1e-9, sum(x[0] for x in kinds.values())), 4)
                          for k, v in kinds.items()},
        # every kernel kind against the HBM copy rate and (GEMMs) the INT8 peak
        "per_kind": {k: {"avg_launch_us": round(1e3 * v[0] / max(1, v[2]), 3),
                         "GB/s": round(v[1] / max(1e-12, v[0] * 1e-3) / 1e9, 1),
                         "frac_hbm": round(v[1] / max(1e-12, v[0] * 1e-3) / 1e9
                                           / peaks["hbm_gbs"], 4),
                         **({"TOP/s": round(v[3] / max(1e-12, v[0] * 1e-3) / 1e12, 1),
                             "frac_int8": round(v[3] / max(1e-12, v[0] * 1e-3) / 1e12 / i8, 4)}
                            if v[3] else {})}
                     for k, v in kinds.items()}})
    rec = {"value": round(value, 4), "ms_per_step": round(ms_per_step, 5), "roofline": roof,
           "gpu_launches": r["launches_per_step"] * steps}
    if "e2e_ms" in r:
        rec["e2e"] = {"value": round(r["ops_step"] * world / (r["e2e_ms"] / steps * 1e-3) / 1e12,
                                     4),
                      "unit": "TOPS", "h2d_bytes_per_step": r["h2d"],
                      "d2h_bytes_per_step": r["d2h"],
                      "ms_per_step": round(r["e2e_ms"] / steps, 5),
                      "how": "per step: one pinned-host -> device copy of every case's X, "
                             "quantize + the GEMMs (CUDA graph), one device -> pinned-host copy "
                             "of every Y; copies of neighbouring steps overlap the kernels (two "
                             "device buffer sets, three streams)"}
    return rec


def workload_config(r, world, norm):
    return {"workload": r["workload"], "description": r["desc"], "cases": r["cases"],
            "activation_pass": ("RMS normalisation (seeded gain ~N(1,0.1), eps 1e-5) "
                                "absorbed into the quantize kernel" if norm else
                                "quantize (amax, threshold, gather, int8)"),
            "mixed_tokens_per_case": r["mixed_tokens"],
            "l2": f"inputs larger than L2: {r['touched'] / 1e6:.0f} MB of distinct weights per "
                  "step (126 MB L2), each case reads its own copy",
            "launch": "one CUDA graph per step (captured once, replayed); kernels chained with "
                      "programmatic dependent launch; step order: all quantize, then all GEMMs "
                      "of each weight format in turn; per-kernel-kind times from graph copies "
                      "with events at the phase boundaries, replayed after the timed steps",
            "parallelism": f"dp{world} (independent batches per GPU, no collective)"}


def run_gpu(args, rank, world):
    import torch

    import mixed_precision_quantized_mixq_b200 as mq

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    gpu_id = None
    try:
        gpu_id = str(torch.cuda.get_device_properties(dev).uuid)
        gpu_id = gpu_id if gpu_id.startswith("GPU-") else "GPU-" + gpu_id
    except Exception:
        gpu_id = None
    sampler = ClockSampler(gpu_id)
    time.sleep(0.3)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    peak_info = {}

    def int8_peak(timed_ms):
        # the INT8 MMA rate loop, just before the timed region and for as long as it
        # (at least 0.2 s), so that both run at the same power and clock state
        secs = min(3.0, max(0.2, timed_ms * 1e-3))
        sampler.mark("int8_peak", True)
        peak_info["i8"] = measure_mma_rate(mq, torch, dev, MMA_I8, secs, st)
        sampler.mark("int8_peak", False)
        peak_info["f16"] = measure_mma_rate(mq, torch, dev, MMA_F16, 0.1, st)
        mq.check_status(st)

    main = measure_workload(mq, torch, dev, rank, world, args.workload, args.modes, args.steps,
                            args.warmup, args.norm, sampler, "main", before_timed=int8_peak,
                            case_filter=args.case)
    i8 = peak_info["i8"]["median"]
    rule = (f"measured in this run: the library's tcgen05.mma kind::i8 rate loop (M=128, N=256, "
            f"K=32 per MMA, operands resident in shared memory, one CTA per SM), median of "
            f"{peak_info['i8']['launches']} launches over {peak_info['i8']['seconds']} s just "
            "before the timed region")
    dec = None
    if not args.no_decode and args.decode_workload != args.workload:
        dsteps = max(200, args.steps)
        dec = measure_workload(mq, torch, dev, rank, world, args.decode_workload, None, dsteps,
                               args.warmup, args.norm, sampler, "decode")
    clocks = sampler.stop()

    rec = build_record(main, world, peaks, peak_src, (i8, rule))
    result = {
        "metric": METRIC, "value": rec["value"], "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": rec["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8 (int8 x int8 -> int32 tensor cores) + fp16 outlier slice (fp32 accumulate)",
        "data": "synthetic (seeded normals; random-init weights of the Llama shapes)",
        "config": workload_config(main, world, args.norm),
        "roofline": rec["roofline"],
        "e2e": rec["e2e"],
        "clocks": clocks.get("main"),
        "gpu_launches": rec["gpu_launches"],
        "tensor_peaks": {
            "int8_rate_loop_tops": {"median": round(i8, 1),
                                    "max": round(peak_info["i8"]["max"], 1),
                                    "clocks": clocks.get("int8_peak")},
            "f16_rate_loop_tflops": round(peak_info["f16"]["median"], 1),
            "bf16_cublas_tflops_measured": {"burst": peaks["bf16_tflops"],
                                            "sustained": peaks["bf16_tflops_sustained"],
                                            "source": peak_src},
        },
    }
    if dec is not None:
        drec = build_record(dec, world, peaks, peak_src, (i8, rule))
        result["decode"] = {"workload": dec["workload"], "value": drec["value"], "unit": "TOPS",
                            "steps": dec["steps"], "ms_per_step": drec["ms_per_step"],
                            "config": workload_config(dec, world, args.norm),
                            "roofline": drec["roofline"], "e2e": drec["e2e"],
                            "clocks": clocks.get("decode"),
                            "gpu_launches": drec["gpu_launches"]}
        result["gpu_launches"] += drec["gpu_launches"]
        result["gpu_launches_note"] = ("kernels of the main timed region plus the decode "
                                       "sub-record's timed region")
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
            W = wraw[(case.N, case.K)]
            Wq8, s_w, W_out = oracle.prepack_w8(W, idx)
            _, _, _, w8eff = oracle.prepack_w4(Wq8)
            entry = {"w8": (Wq8, s_w, W_out), "w4": (w8eff, s_w, W_out)}
            if "w4b" in modes:
                entry["w4b"] = (oracle.prepack_w4b(W), W_out)
            wcache[key] = entry
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
    xo = X_out if X_out.shape[1] else None
    ops = 0
    for mode in modes:
        if mode == "w4b":
            (q, s, z), W_out = w["w4b"]
            wo = W_out if W_out.shape[1] else None
            oracle.linear_w4b_points(Xq, s_x, xo, q, s, z, wo, ms, ns)
        else:
            Wq, s_w, W_out = w[mode]
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


def _sample_text(units, points, cases, modes):
    return (f"{units} units of (one token of one case, quantize + "
            f"{' + '.join(MODE_NAMES[m].split(' ')[0] + ('b' if m == 'w4b' else '') for m in modes)}"
            f" at {points} sampled output channels), cycling over the {cases} cases; plain C "
            "oracle, OpenMP over outputs")


def run_cpu_baseline(args, budget_s=15.0, workload=None, modes=None):
    workload = workload or args.workload
    _, cases = workload_cases(workload, args.case, modes or args.modes)
    points = 2048
    sampler = OracleSampler(oracle_prepare(cases, args.norm), points)
    units = calibrate(sampler, budget_s)
    t0 = time.perf_counter()
    ops = sampler.run(units)
    dt = time.perf_counter() - t0
    return {"value": round(ops / dt / 1e12, 6), "unit": "TOPS", "cores": cpu_cores(points),
            "kind": "oracle",
            "sample": _sample_text(units, points, len(sampler.prepared), cases[0][1])
                      + f"; workload {workload}; {dt:.1f} s"}


def single_core_baselines(budget_s=6.0):
    """The oracle on one host core (OMP_NUM_THREADS=1, a child process) for the tiny and
    the decode workloads."""
    out = {}
    for w in ("tiny", "llama7b-decode"):
        env = dict(os.environ, OMP_NUM_THREADS="1")
        cmd = [sys.executable, os.path.abspath(__file__), "--single-core-probe", w,
               "--probe-seconds", str(budget_s)]
        try:
            p = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=300)
            out[w] = json.loads(p.stdout.strip().splitlines()[-1])
        except Exception as e:  # reported, not fatal: the baseline is context only
            out[w] = {"error": f"{type(e).__name__}: {e}"[:200]}
    return out


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle on the host cores, same metric and workload; each step
    is a bounded sample sized so the whole run takes about a minute."""
    if rank != 0:
        return None
    desc, cases = workload_cases(args.workload, args.case, args.modes)
    points = 2048
    sampler = OracleSampler(oracle_prepare(cases, getattr(args, "norm", False)), points)
    step_s = min(0.5, 60.0 / (args.steps + args.warmup))
    units = calibrate(sampler, step_s)
    sampler.run(units * args.warmup)
    t0 = time.perf_counter()
    ops = sampler.run(units * args.steps)
    dt = time.perf_counter() - t0
    value = ops / dt / 1e12
    sample = "per step: " + _sample_text(units, points, len(cases), cases[0][1])
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
    argv = list(sys.argv[1:] if argv is None else argv)
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama7b-prefill", choices=WORKLOADS)
    ap.add_argument("--decode-workload", default="llama7b-decode", choices=WORKLOADS,
                    help="workload of the small-M (HBM-bound) sub-record")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode sub-record")
    ap.add_argument("--impl", default="mixq", choices=["mixq", "reference"])
    ap.add_argument("--case", default=None, help="keep only cases whose name contains this")
    ap.add_argument("--modes", default=None,
                    help="weight formats of the main workload: w8, w4, w4b (comma separated)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--norm", action="store_true",
                    help="absorb an RMS normalisation of each token (seeded gain ~N(1,0.1), "
                         "eps 1e-5) into the activation pass")
    ap.add_argument("--single-core-probe", default=None, help=argparse.SUPPRESS)
    ap.add_argument("--probe-seconds", type=float, default=6.0, help=argparse.SUPPRESS)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3

    if args.single_core_probe:
        r = run_cpu_baseline(args, budget_s=args.probe_seconds, workload=args.single_core_probe)
        print(json.dumps(r), flush=True)
        return 0

    world_env = os.environ.get("WORLD_SIZE")
    if world_env is None and args.gpus > 1:
        return launch_ranks(args.gpus, argv)
    world = int(world_env or "1")
    rank = int(os.environ.get("RANK", "0"))
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but the launcher started {world} ranks",
              file=sys.stderr)
        return 2
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
        res["cpu_baseline"]["single_core"] = single_core_baselines()
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
