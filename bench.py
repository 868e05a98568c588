#!/usr/bin/env python
"""Benchmark of the FP8 W8A8 linear hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the path over one batch already resident in HBM:
per-token dynamic E4M3 quantization of the activations followed by the FP8
tcgen05 GEMM with the fused dequantization / FP16 epilogue (for the MoE
workload: quantize -> grouped up GEMM -> re-quantize -> grouped down GEMM).
Weights are quantized once, offline, outside the timed region.

Default workload: the dense FFN pair, the largest single-GPU configuration:
up X fp16 [8192, 2048] times W1 [8192, 2048] and down X fp16 [8192, 8192]
times W2 [2048, 8192] (0.5% outlier channels x30), both linears per step.
--workload qkv|tiny|ffn_up|ffn_down|moe|moe_tokens|sweep_mM selects another.
Metric: TFLOP/s = sum of 2*M*N*K per step / time.  L2 is defeated by rotating
through enough independent copies of every input and output that one
rotation is more than 3x the 126 MB L2.

Tensor-bound fractions are reported against 2 x the measured bf16 GEMM peak
(the fp8/bf16 nominal ratio) and against an FP8 ceiling measured in the same
run: torch._scaled_mm (a library GEMM, E4M3 x E4M3, row-wise scales) at
8192^3, best of 10 by CUDA events.

Multi-GPU (torchrun, one process per GPU): independent replicas, no
data-path collective; each rank runs the same number of steps on its own
buffers, time = max over ranks, value = all ranks' FLOPs / that time.

--impl reference times the CPU oracle (oracle/, NumPy, float64) on the host
cores on a bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import signal
import statistics
import subprocess
import sys
import tempfile
import time
from datetime import timedelta

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from fp8_quantized_generative_b200 import workloads as wl  # noqa: E402

METRIC = "FP8 W8A8 linear TFLOPS (quant+GEMM+dequant) and % of B200 FP8 / HBM roofline"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0   # nominal dense ratio 4.5 / 2.25 PFLOP/s


# --------------------------------------------------------------------------- workloads
def workload_spec(name: str):
    """Return (description, kind, tensors) for a named workload; tensors are CPU fp16."""
    # dense workloads: a list of (X, W) linears, all run in every step
    if name == "ffn":
        up, down = wl.ffn()
        return ("ffn_pair up M=8192 N=8192 K=2048 + down M=8192 N=2048 K=8192 (independent inputs)", "dense",
                [(up.X, up.W), (down.X, down.W)])
    if name == "qkv":
        lin = wl.qkv()
        return "qkv_projection M=4096 N=6144 K=2048", "dense", [(lin.X, lin.W)]
    if name == "tiny":
        lin = wl.tiny()
        return "tiny_linear M=32 N=256 K=256", "dense", [(lin.X, lin.W)]
    if name in ("ffn_up", "ffn_down"):
        up, down = wl.ffn()
        lin = up if name == "ffn_up" else down
        M, K = lin.X.shape
        return f"{name} M={M} N={lin.W.shape[0]} K={K}", "dense", [(lin.X, lin.W)]
    if name.startswith("sweep_m"):
        m = int(name[len("sweep_m"):])
        lin = wl.sweep(m)
        return f"square_linear M={m} N=4096 K=4096", "dense", [(lin.X, lin.W)]
    if name == "moe":
        m = wl.moe()
        return ("moe_ffn T=8192 top2 E=64 d=2048 F=1024 (16384 grouped rows)", "moe",
                (m.X_perm, m.offsets, m.W_up, m.W_down))
    if name == "moe_tokens":
        # the same layer from and back to the token matrix: tokens quantized
        # once, the up projection gathers its rows by the router's grouping and
        # the down projection adds each row, weighted, into its token (combine)
        m = wl.moe()
        return ("moe_ffn T=8192 top2 E=64 d=2048 F=1024 from and back to the 8192-token matrix "
                "(dispatch to the expert rows, weighted top-2 combine)", "moe",
                (m.X, m.offsets, m.W_up, m.W_down, np.asarray(m.token_of_row, dtype=np.int32),
                 np.asarray(m.row_weight, dtype=np.float32)))
    raise SystemExit(f"unknown workload {name}")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.send_signal(signal.SIGTERM)
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return self.summarize(lines)

    @staticmethod
    def summarize(lines):
        """Median SM clock, the highest max clock and every throttle reason
        seen active, from nvidia-smi CSV lines in FIELDS order (lines that do
        not parse are skipped)."""
        rows = []
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags in rows for i, v in enumerate(flags) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------- GPU arm
class Plan:
    """Device buffers (rotated sets) and the raw C-ABI launch sequence of one step."""

    def __init__(self, kind, tensors, device, min_rotation_bytes, fused=True, x_fmt="e4m3", weights="channel",
                 dispatch="quant", overlap=False):
        import fp8_quantized_generative_b200 as fq
        from fp8_quantized_generative_b200 import _lib
        self.fq, self.L = fq, _lib
        self.kind = kind
        self.device = device
        # activation codes E4M3 (the path) or E5M2 (variant); weight scales per channel or per tensor (variant)
        self.x_fmt = x_fmt
        # per-tensor scales: the dense (FFN) variant; 128x128 block scales: the MoE variant
        if (weights == "tensor" and kind != "dense") or (weights == "block" and kind == "dense"):
            raise SystemExit(f"--weight-scales {weights} applies to "
                             f"{'dense' if weights == 'tensor' else 'moe'} workloads only")
        if kind != "dense" and len(tensors) > 4 and (weights != "channel" or x_fmt != "e4m3"):
            raise SystemExit("the row-gather / combine MoE form runs E4M3 activations with per-channel weights")
        self.weights = weights
        self.fmt = _lib.FORMATS[x_fmt]
        if kind == "dense":
            # one or more linears per step: (M, N, K) of each
            self.shapes = [(X.shape[0], W.shape[0], X.shape[1]) for X, W in tensors]
            Ms = [m for m, _, _ in self.shapes]
            # Up to 16 token rows the library quantizes inside the GEMM (one launch; E4M3 only).
            self.fused = fused and x_fmt == "e4m3" and max(Ms) <= fq.FUSED_MAX_ROWS
            # More than 128 rows: one launch that quantizes inside the CTA-pair GEMM (E4M3 only).
            self.overlap = overlap and x_fmt == "e4m3" and min(Ms) > 128
            self.flops = sum(2.0 * M * N * K for M, N, K in self.shapes)
            per_set = sum(M * K * 3 + 4 * M + N * K + 4 * N + 2 * M * N for M, N, K in self.shapes)
        else:
            self.fused = self.overlap = False
            Xp, offsets, Wu, Wd = tensors[:4]
            # gather form: Xp is the token matrix and tensors[4] the row -> token map
            self.row_token = tensors[4] if len(tensors) > 4 else None
            self.row_weight = tensors[5] if len(tensors) > 5 else None   # and the combine weights
            # token -> grouped rows by the quantizer's store (quant), or grouped rows <- tokens by the GEMM (gemm)
            self.dispatch = dispatch if self.row_token is not None else None
            self.gather = self.dispatch == "gemm"
            self.T = Xp.shape[0]
            self.R = int(offsets[-1])
            self.D = Xp.shape[1]
            self.E, self.F, _ = Wu.shape
            self.flops = 2.0 * self.R * self.F * self.D * 2
            self.out_rows = self.T if self.row_weight is not None else self.R
            per_set = (self.T * self.D * 3 + 8 * self.R + 2 * self.E * self.F * self.D + 8 * self.E * self.F
                       + self.R * self.F * 5 + self.out_rows * self.D * 2 + 4 * self.R)
        self.sets = max(2, math.ceil(min_rotation_bytes / per_set))
        self.bufs = []
        for i in range(self.sets):
            b = {}
            if kind == "dense":
                qw = fq.quantize_weight_per_tensor if weights == "tensor" else fq.quantize_weight_per_channel
                for l, ((X, W), (M, N, K)) in enumerate(zip(tensors, self.shapes)):
                    b[f"X{l}"] = X.to(device)
                    b[f"Wq{l}"], b[f"sw{l}"] = qw(W.to(device))
                    b[f"Xq{l}"] = torch.empty((M, K), dtype=torch.uint8, device=device)
                    b[f"sx{l}"] = torch.empty((M,), dtype=torch.float32, device=device)
                    b[f"Y{l}"] = torch.empty((M, N), dtype=torch.float16, device=device)
                    if self.overlap:
                        b[f"sync{l}"] = torch.zeros((int(_lib.fp8q_overlap_sync_words(M)),), dtype=torch.int32,
                                                    device=device)
            else:
                b["X"] = Xp.to(device)
                b["off"] = torch.from_numpy(offsets).to(device)
                if self.row_token is not None:
                    b["rt"] = torch.from_numpy(self.row_token).to(device)
                if self.dispatch == "quant":
                    b["tr"] = torch.from_numpy(wl.token_rows(self.row_token, self.T)).to(device)
                if self.row_weight is not None:
                    b["rw"] = torch.from_numpy(self.row_weight).to(device)
                qw = fq.quantize_weight_blockwise if weights == "block" else fq.quantize_weight_per_channel
                b["Wuq"], b["swu"] = qw(Wu.to(device))
                b["Wdq"], b["swd"] = qw(Wd.to(device))
                xrows = self.R if self.dispatch == "quant" else self.T   # quantized rows: grouped or tokens
                b["Xq"] = torch.empty((xrows, self.D), dtype=torch.uint8, device=device)
                b["sx"] = torch.empty((xrows,), dtype=torch.float32, device=device)
                b["H"] = torch.empty((self.R, self.F), dtype=torch.float16, device=device)
                b["Hq"] = torch.empty((self.R, self.F), dtype=torch.uint8, device=device)
                b["sh"] = torch.empty((self.R,), dtype=torch.float32, device=device)
                b["Y"] = torch.empty((self.out_rows, self.D), dtype=torch.float16, device=device)
            b = {k: v for k, v in b.items()}
            b["p"] = {k: v.data_ptr() for k, v in b.items()}
            self.bufs.append(b)
        torch.cuda.synchronize(device)
        self.bytes_per_set = per_set
        self.kernels = self._kernel_names()
        self.launches_per_step = len(self.kernels)

    def _kernel_names(self):
        if self.kind == "dense":
            # (layer, op) of each launch of a step; op: "fused", "overlap", "quant" or "gemm"
            tag = (lambda l: "") if len(self.shapes) == 1 else (lambda l: ("_up", "_down")[l] if len(self.shapes) == 2
                                                                  else f"_{l}")
            ops = ["fused"] if self.fused else ["overlap"] if self.overlap else ["quant", "gemm"]
            self.dense_launches = [(l, op) for l in range(len(self.shapes)) for op in ops]
            name = {"fused": "fp8_quantized_linear_fused", "overlap": "fp8_quantized_linear_overlapped",
                    "quant": "quant_rows", "gemm": "fp8_gemm"}
            return [name[op] + tag(l) for l, op in self.dense_launches]
        up = "fp8_grouped_gemm_up_gather" if self.gather else "fp8_grouped_gemm_up"
        down = "fp8_grouped_gemm_down_combine" if self.row_weight is not None else "fp8_grouped_gemm_down"
        quant = "quant_rows_dispatch" if self.dispatch == "quant" else "quant_rows"
        return [quant, up, "quant_rows_h", down]

    def kernel_bytes_flops(self):
        """Algorithmic bytes and FLOPs of each launch of one step."""
        if self.kind == "dense":
            out = []
            for l, op in self.dense_launches:
                M, N, K = self.shapes[l]
                if op in ("fused", "overlap"):
                    out.append((2 * M * K + N * K + 4 * N + 2 * M * N, 2.0 * M * N * K))
                elif op == "quant":
                    out.append((M * K * 3 + 4 * M, 0.0))
                else:
                    out.append((M * K + N * K + 4 * M + 4 * N + 2 * M * N, 2.0 * M * N * K))
            return out
        R, D, F, E = self.R, self.D, self.F, self.E
        if self.weights == "block":   # one scale per 128 x 128 weight block
            su, sd = 4 * E * (-(-F // 128)) * (-(-D // 128)), 4 * E * (-(-D // 128)) * (-(-F // 128))
        else:
            su, sd = 4 * E * F, 4 * E * D
        # dispatch: each token read once and written to its grouped rows (+ the token -> row map)
        q0 = ((self.T * D * 2 + R * D + 4 * R + 4 * self.T * 2, 0.0) if self.dispatch == "quant"
              else (self.T * D * 3 + 4 * self.T, 0.0))
        return [q0,
                (R * D + E * F * D + 4 * R + su + 2 * R * F, 2.0 * R * F * D),
                (R * F * 3 + 4 * R, 0.0),
                (R * F + E * D * F + 4 * R + sd + 2 * R * D, 2.0 * R * D * F) if self.row_weight is None else
                # combine: + token index and weight per row; the output is the [T, D] token matrix
                (R * F + E * D * F + 12 * R + sd + 2 * self.T * D, 2.0 * R * D * F)]

    def launch(self, i, k):
        """Launch kernel k of step i (raw C ABI, integer pointers)."""
        L, p = self.L, self.bufs[i % self.sets]["p"]
        st = torch.cuda.current_stream(self.device).cuda_stream   # the capture stream inside a graph
        if self.kind == "dense":
            l, op = self.dense_launches[k]
            M, N, K = self.shapes[l]
            X, Wq, sw, Xq, sx, Y = (p[f"{n}{l}"] for n in ("X", "Wq", "sw", "Xq", "sx", "Y"))
            if op == "fused":
                s = L.fp8q_quantized_linear(X, Wq, sw, M, N, K, Y, 0, 0, st)
            elif op == "overlap":
                s = L.fp8q_quantized_linear_overlapped(X, Wq, sw, M, N, K, Y, Xq, sx, p[f"sync{l}"], st)
            elif op == "quant":
                s = L.fp8q_quantize_rows_dynamic_fmt(X, M, K, self.fmt, Xq, sx, st)
            else:
                s = L.fp8q_linear_fmt(Xq, self.fmt, sx, Wq, sw, M, N, K, Y, st)
        else:
            if k == 0 and self.dispatch == "quant":
                s = L.fp8q_quantize_rows_dispatch(p["X"], self.T, self.D, self.fmt, p["tr"], 2, self.R, p["Xq"],
                                                  p["sx"], st)
            elif k == 0:
                s = L.fp8q_quantize_rows_dynamic_fmt(p["X"], self.T, self.D, self.fmt, p["Xq"], p["sx"], st)
            elif k == 1 and self.gather:
                s = L.fp8q_moe_grouped_linear_gather(p["Xq"], p["sx"], self.T, p["rt"], p["off"], self.E, self.R,
                                                     p["Wuq"], p["swu"], self.F, self.D, p["H"], st)
            elif k == 1:
                if self.weights == "block":
                    s = L.fp8q_moe_grouped_linear_blockscaled(p["Xq"], p["sx"], p["off"], self.E, self.R, p["Wuq"],
                                                              p["swu"], self.F, self.D, p["H"], st)
                else:
                    s = L.fp8q_moe_grouped_linear_fmt(p["Xq"], self.fmt, p["sx"], p["off"], self.E, self.R,
                                                      p["Wuq"], p["swu"], self.F, self.D, p["H"], st)
            elif k == 2:
                s = L.fp8q_quantize_rows_dynamic_fmt(p["H"], self.R, self.F, self.fmt, p["Hq"], p["sh"], st)
            elif self.row_weight is not None:
                s = L.fp8q_moe_grouped_linear_combine(p["Hq"], p["sh"], p["off"], self.E, self.R, p["Wdq"], p["swd"],
                                                      self.D, self.F, p["rt"], p["rw"], self.T, p["Y"], st)
            elif self.weights == "block":
                s = L.fp8q_moe_grouped_linear_blockscaled(p["Hq"], p["sh"], p["off"], self.E, self.R, p["Wdq"],
                                                          p["swd"], self.D, self.F, p["Y"], st)
            else:
                s = L.fp8q_moe_grouped_linear_fmt(p["Hq"], self.fmt, p["sh"], p["off"], self.E, self.R, p["Wdq"],
                                                  p["swd"], self.D, self.F, p["Y"], st)
        if s != 0:
            L.check(s, f"launch {self.kernels[k]}")

    def step(self, i):
        for k in range(self.launches_per_step):
            self.launch(i, k)


def _graph_of(plan, launches):
    """Capture the (step, kernel) launches into a CUDA graph and upload it."""
    dev = plan.device
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(device=dev)
    cap.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.graph(g, stream=cap):
        for i, k in launches:
            plan.launch(i, k)
    torch.cuda.synchronize(dev)
    g.replay()
    torch.cuda.synchronize(dev)
    return g


def timed_gpu(plan, steps, barrier, use_graph=True):
    """Time exactly `steps` steps of the path.

    With use_graph the steps are captured once into a CUDA graph (launch
    overhead removed, as a serving loop would run them); the graph is
    replayed once untimed to upload it, then the timed replay is bracketed by
    CUDA events on the replay stream.  Each kernel's own duration is timed the
    same way from a graph holding only that kernel's launches of the same
    steps (events recorded inside a graph cannot be timed).
    """
    dev = plan.device
    nk = plan.launches_per_step
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if not use_graph:
        ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nk)]
              for _ in range(steps)]
        barrier()
        torch.cuda.synchronize(dev)
        t0.record()
        for i in range(steps):
            for k in range(nk):
                ev[i][k][0].record()
                plan.launch(i, k)
                ev[i][k][1].record()
        t1.record()
        torch.cuda.synchronize(dev)
        barrier()
        per_kernel_ms = [statistics.fmean(ev[i][k][0].elapsed_time(ev[i][k][1]) for i in range(steps))
                         for k in range(nk)]
        return t0.elapsed_time(t1), per_kernel_ms

    g = _graph_of(plan, [(i, k) for i in range(steps) for k in range(nk)])
    barrier()
    torch.cuda.synchronize(dev)
    t0.record()
    g.replay()
    t1.record()
    torch.cuda.synchronize(dev)
    barrier()
    total_ms = t0.elapsed_time(t1)
    del g
    per_kernel_ms = []
    for k in range(nk):
        gk = _graph_of(plan, [(i, k) for i in range(steps)])
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        gk.replay()
        b.record()
        torch.cuda.synchronize(dev)
        per_kernel_ms.append(a.elapsed_time(b) / steps)
        del gk
    return total_ms, per_kernel_ms


def timed_e2e(plan, tensors, steps):
    """Host-buffer path through the public C ABI, every step: pinned H2D of
    the step's activations, the library calls, D2H of the step's outputs.
    Steps alternate over two streams with their own buffers, so one step's
    D2H overlaps the next step's H2D and kernels (PCIe is full duplex); the
    timed region is bracketed by events on the launching stream."""
    dev = plan.device
    main = torch.cuda.current_stream(dev)
    streams = [torch.cuda.Stream(device=dev) for _ in range(2)]
    if plan.kind == "dense":
        ins = [(X, f"X{l}") for l, (X, _) in enumerate(tensors)]
        outs = [f"Y{l}" for l in range(len(tensors))]
    else:
        ins, outs = [(tensors[0], "X")], ["Y"]
    xh = [(X.pin_memory(), key) for X, key in ins]
    yh = [[torch.empty(tuple(plan.bufs[0][key].shape), dtype=torch.float16).pin_memory() for key in outs]
          for _ in range(2)]
    h2d = sum(x.numel() * x.element_size() for x, _ in xh)
    d2h = sum(y.numel() * y.element_size() for y in yh[0])

    def one(i):
        j = i % 2
        with torch.cuda.stream(streams[j]):
            b = plan.bufs[j % plan.sets]
            for x, key in xh:
                b[key].copy_(x, non_blocking=True)
            plan.step(j)
            for y, key in zip(yh[j], outs):
                y.copy_(b[key], non_blocking=True)

    for i in range(2):
        one(i)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(main)
    for st in streams:
        st.wait_event(t0)
    for i in range(steps):
        one(i)
    for st in streams:
        main.wait_stream(st)
    t1.record(main)
    torch.cuda.synchronize(dev)
    return t0.elapsed_time(t1), h2d, d2h


def fp8_ceiling(device, n=8192, reps=10):
    """FP8 tensor-core ceiling measured with a library GEMM: torch._scaled_mm,
    E4M3 x E4M3 at n^3 with row-wise fp32 scales and bf16 output (tensor-wise
    scales if row-wise is not supported), best of `reps` by CUDA events after
    warm-up.  Returns (TFLOP/s, description) or (None, reason)."""
    try:
        g = torch.Generator(device=device).manual_seed(7)
        a = torch.randn((n, n), device=device, generator=g).to(torch.float8_e4m3fn)
        b = torch.randn((n, n), device=device, generator=g).to(torch.float8_e4m3fn).t()   # column-major
        forms = [("row-wise scales", torch.ones((n, 1), device=device), torch.ones((1, n), device=device)),
                 ("tensor-wise scales", torch.ones((), device=device), torch.ones((), device=device))]
        for what, sa, sb in forms:
            try:
                torch._scaled_mm(a, b, scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16)
            except (RuntimeError, TypeError):
                continue
            for _ in range(5):
                torch._scaled_mm(a, b, scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16)
            best = float("inf")
            for _ in range(reps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                torch._scaled_mm(a, b, scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16)
                e1.record()
                torch.cuda.synchronize(device)
                best = min(best, e0.elapsed_time(e1))
            return 2.0 * n ** 3 / (best * 1e-3) / 1e12, (f"torch._scaled_mm {n}^3 E4M3 x E4M3, {what}, bf16 out, "
                                                         f"best of {reps} ({best * 1e3:.1f} us)")
        return None, "torch._scaled_mm rejected both scale forms"
    except Exception as e:   # a measurement aid only: the bench line still stands without it
        return None, f"torch._scaled_mm failed: {type(e).__name__}: {e}"


# --------------------------------------------------------------------------- oracle arm
def oracle_sampler(kind, tensors, m_rows, n_rows, x_fmt="e4m3", weights="channel"):
    """A callable running the oracle on an (m_rows x n_rows) output sample; returns its FLOPs."""
    from oracle import linear_blockscaled_ref, linear_ref, moe_combine_ref, quant_blocks, quant_rows, quant_tensor
    if kind == "dense":
        layers = []
        for X, W in tensors:
            Xn = X.numpy()
            # offline weight quantization, untimed
            Wq, sw = quant_tensor(W.numpy()) if weights == "tensor" else quant_rows(W.numpy())
            layers.append((Xn, Wq, sw, min(m_rows, Xn.shape[0]), min(n_rows, Wq.shape[0])))
        state = {"i": 0}

        def run():
            i = state["i"]
            state["i"] += 1
            flops = 0.0
            for Xn, Wq, sw, mr, nr in layers:
                r0 = (i * mr) % max(1, Xn.shape[0] - mr + 1)
                c0 = (i * nr) % max(1, Wq.shape[0] - nr + 1)
                xq, sx = quant_rows(Xn[r0:r0 + mr], x_fmt)
                linear_ref(xq, sx, Wq[c0:c0 + nr], sw[c0:c0 + nr], x_fmt)
                flops += 2.0 * mr * nr * Xn.shape[1]
            return flops
        return run, "; ".join(f"{mr} activation rows x {nr} weight rows (output block) of the {Xn.shape[0]}x"
                              f"{Wq.shape[0]}x{Xn.shape[1]} linear" for Xn, Wq, _, mr, nr in layers) + " per call"
    Xp, offsets, Wu, Wd = tensors[:4]
    e = int(np.argmax(np.diff(offsets)))
    lo = int(offsets[e])
    cnt = min(m_rows, int(offsets[e + 1]) - lo)
    # gather form: the expert's rows are tokens row_token[lo:lo+cnt]
    Xn = Xp.numpy()[tensors[4][lo:lo + cnt]] if len(tensors) > 4 else Xp.numpy()[lo:lo + cnt]
    D = Xn.shape[1]
    if weights == "block":
        Wuq, swu = quant_blocks(Wu[e].numpy()[:n_rows])
        Wdq, swd = quant_blocks(Wd[e].numpy()[:n_rows, :n_rows])

        def run():
            xq, sx = quant_rows(Xn)
            h = linear_blockscaled_ref(xq, sx, Wuq, swu)
            hq, sh = quant_rows(h)
            linear_blockscaled_ref(hq, sh, Wdq, swd)
            return 2.0 * cnt * Wuq.shape[0] * D + 2.0 * cnt * n_rows * hq.shape[1]
        return run, (f"expert {e}: {cnt} rows through up ({n_rows} channels) and down ({n_rows} channels), "
                     "128x128 block-scaled weights")
    Wuq, swu = quant_rows(Wu[e].numpy()[:n_rows])
    Wdq, swd = quant_rows(Wd[e].numpy()[:, :])

    if len(tensors) > 5:
        # combine form: the down projection adds each weighted row into its token
        # (one row per token within one expert, so the sample's tokens are local)
        rw = np.asarray(tensors[5][lo:lo + cnt], dtype=np.float32)
        one = np.array([0, cnt], dtype=np.int64)
        local = np.arange(cnt)

        def down(hq, sh):
            moe_combine_ref(hq, sh, one, Wdq[None, :n_rows, :hq.shape[1]], swd[None, :n_rows], local, rw, cnt)
    else:
        def down(hq, sh):
            # down projection restricted to the sampled hidden columns
            linear_ref(hq, sh, Wdq[:n_rows, :hq.shape[1]], swd[:n_rows], x_fmt)

    def run():
        xq, sx = quant_rows(Xn, x_fmt)
        h = linear_ref(xq, sx, Wuq, swu, x_fmt)
        hq, sh = quant_rows(h, x_fmt)
        down(hq, sh)
        return 2.0 * cnt * Wuq.shape[0] * D + 2.0 * cnt * n_rows * hq.shape[1]
    return run, (f"expert {e}: {cnt} rows through up ({n_rows} channels) and down ({n_rows} channels)"
                 + (", weighted combine into the rows' tokens" if len(tensors) > 5 else ""))


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(kind, tensors, budget_s=10.0, x_fmt="e4m3", weights="channel"):
    run, sample = oracle_sampler(kind, tensors, 64, 6144 if kind == "dense" else 1024, x_fmt, weights)
    run()                                           # warm (page-in, BLAS threads)
    flops, t0 = 0.0, time.perf_counter()
    while True:
        flops += run()
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": flops / el / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{sample}; repeated for {el:.1f} s", "seconds": round(el, 2)}


# --------------------------------------------------------------------------- main
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not torch.distributed.is_initialized():
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=timedelta(seconds=120))
    return world, rank, local


def make_barrier(world, device):
    if world == 1:
        return lambda: None

    def barrier():
        if device is not None and device.type == "cuda":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()
    return barrier


def replica_value(flops_per_step: float, steps: int, world: int, t_max_ms: float) -> float:
    """Whole-job TFLOP/s of `world` independent replicas each running `steps`
    steps: every rank's FLOPs over the slowest rank's time."""
    return flops_per_step * steps * world / (t_max_ms * 1e-3) / 1e12


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def run_reference(args, world, rank):
    if rank != 0:
        return None
    desc, kind, tensors = workload_spec(args.workload)
    run, sample = oracle_sampler(kind, tensors, 32, 256, args.x_fmt, args.weight_scales)
    for _ in range(args.warmup):
        run()
    flops, t0 = 0.0, time.perf_counter()
    for _ in range(args.steps):
        flops += run()
    el = time.perf_counter() - t0
    value = flops / el / 1e12
    cores = blas_threads()
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": desc, "sample_per_step": sample, "parallelism": "host cores (rank 0 only)",
                       "activation_format": args.x_fmt,
                       "weight_scales": "per-" + args.weight_scales},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_ours(args, world, rank, local):
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for --impl ours")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    barrier = make_barrier(world, device)
    desc, kind, tensors = workload_spec(args.workload)
    import fp8_quantized_generative_b200 as fq
    fq.set_gemm_tuning({"auto": 0, "single": 1, "pair": 2, "splitk": 3}[args.gemm], args.bn, args.ksplit)
    plan = Plan(kind, tensors, device, min_rotation_bytes=3 * L2_BYTES, fused=args.fused, x_fmt=args.x_fmt,
                dispatch=args.dispatch, overlap=args.overlap,
                weights=args.weight_scales)
    peaks, peak_src = load_peaks()
    ceiling, ceiling_how = fp8_ceiling(device)

    sampler = ClockSampler(local)
    for i in range(args.warmup):
        plan.step(i)
    torch.cuda.synchronize(device)
    sampler.start()
    time.sleep(0.2)
    total_ms, per_kernel_ms = timed_gpu(plan, args.steps, barrier, use_graph=not args.no_graph)
    clocks = sampler.stop()
    flag = plan.fq.device_error()
    if flag:
        raise SystemExit(f"device error word 0x{flag:x} after the timed region")

    t_max_ms = max_over_ranks(total_ms, world, device)
    value = replica_value(plan.flops, args.steps, world, t_max_ms)

    e2e_steps = max(3, min(args.steps, 50))
    e2e_ms, h2d, d2h = timed_e2e(plan, tensors, e2e_steps)
    e2e_ms = max_over_ranks(e2e_ms, world, device)
    e2e_value = replica_value(plan.flops, e2e_steps, world, e2e_ms)

    # roofline of each kernel; the dominant one (largest time share) is reported as "roofline"
    bf = plan.kernel_bytes_flops()
    hbm = float(peaks["hbm_gbs"])
    # A tensor-bound kernel timed over a seconds-long back-to-back loop runs
    # under the 1 kW power cap: compare it with the sustained GEMM figure; a
    # loop under a second with the burst figure.
    sustained = max(per_kernel_ms) * args.steps > 1000.0 and "bf16_tflops_sustained" in peaks
    bf16 = float(peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"])
    fp8_peak = bf16 * FP8_OVER_BF16
    kern = {}
    for name, ms, (byt, fl) in zip(plan.kernels, per_kernel_ms, bf):
        t_c = fl / (fp8_peak * 1e12) if fl else 0.0
        t_m = byt / (hbm * 1e9)
        bound = "tensor" if t_c > t_m else "hbm"
        if bound == "tensor":
            ach, peak, unit = fl / (ms * 1e-3) / 1e12, fp8_peak, "TFLOP/s"
        else:
            ach, peak, unit = byt / (ms * 1e-3) / 1e9, hbm, "GB/s"
        kern[name] = {"bound": bound, "achieved": round(ach, 2), "peak": round(peak, 1), "unit": unit,
                      "frac": round(ach / peak, 4), "us_per_launch": round(ms * 1e3, 3),
                      "algorithmic_bytes": int(byt), "flops": fl,
                      "gb_s": round(byt / (ms * 1e-3) / 1e9, 1),
                      "tflop_s": round(fl / (ms * 1e-3) / 1e12, 1) if fl else 0.0}
        if bound == "tensor" and ceiling:
            kern[name]["frac_vs_fp8_ceiling"] = round(ach / ceiling, 4)
    dom = max(kern, key=lambda k: kern[k]["us_per_launch"])
    traffic = load_traffic(dom, args.workload)
    d = kern[dom]
    roofline = {"bound": d["bound"], "achieved": d["achieved"], "peak": d["peak"], "unit": d["unit"],
                "frac": d["frac"], "traffic": traffic, "kernel": dom,
                "peak_source": (f"{peak_src} (fp8 = 2 x bf16 {'sustained' if sustained else 'burst'}; "
                                f"timed loop {max(per_kernel_ms) * args.steps:.1f} ms)" if d["bound"] == "tensor"
                                else f"{peak_src} (HBM copy)")}
    if d["bound"] == "tensor":
        roofline["fp8_ceiling"] = {"value": round(ceiling, 1) if ceiling else None, "unit": "TFLOP/s",
                                   "how": ceiling_how,
                                   "frac": round(d["achieved"] / ceiling, 4) if ceiling else None}
    step_flops = plan.flops
    step_bytes = sum(b for b, _ in bf)
    ms_step = t_max_ms / args.steps
    return {"metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": ("fp8e4m3" if args.x_fmt == "e4m3" else "fp8 e5m2 activations x e4m3 weights")
                     + " (fp32 accumulate, fp16 out)",
            "data": "synthetic",
            "config": {"workload": desc, "parallelism": f"replicas x{world} (no collective)",
                       "gemm": args.gemm, "bn": args.bn, "ksplit": args.ksplit,
                       "activation_format": args.x_fmt, "weight_scales": "per-" + plan.weights,
                       "l2": f"rotating {plan.sets} buffer sets of {plan.bytes_per_set / 1e6:.0f} MB "
                             f"(> 3x 126 MB L2), no flush",
                       "step": " -> ".join(plan.kernels),
                       "fused": plan.fused, "overlap": plan.overlap,
                       "launch": "per-call from the host" if args.no_graph else
                                 "CUDA graph of the K timed steps (replayed once untimed to upload)",
                       "kernel_timing": "per-kernel: CUDA events around a graph of that kernel's K launches"
                                        if not args.no_graph else "per-kernel: CUDA events around each launch"},
            "roofline": roofline, "kernels": kern,
            "step_gb_s": round(step_bytes / (ms_step * 1e-3) / 1e9, 1),
            "pct_fp8_peak_step": round(100 * step_flops / (ms_step * 1e-3) / 1e12 / fp8_peak, 2),
            "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "gpu_launches": plan.launches_per_step * args.steps,
            "clocks": clocks}


def csrc_hash() -> str:
    """Hash of the kernel sources (the build whose DRAM counters are committed)."""
    import hashlib
    d = os.path.join(ROOT, "fp8_quantized_generative_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(d)):
        if f.endswith((".cu", ".cuh")):
            h.update(f.encode())
            with open(os.path.join(d, f), "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()[:16]


def load_traffic(kernel, workload):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, or
    None when there is none for this workload or the kernels changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        with open(path) as f:
            t = json.load(f)
        if t.get("csrc_sha256_16") != csrc_hash():
            return None
        return t.get(workload, {}).get(kernel)
    except (OSError, ValueError):
        return None


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="ffn")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dispatch", default="quant", choices=["quant", "gemm"],
                    help="moe_tokens: tokens reach their expert-grouped rows through the quantizer's store "
                         "(quant) or through the up GEMM's row gather (gemm)")
    ap.add_argument("--no-graph", action="store_true", help="launch every step from the host instead of a CUDA graph")
    ap.add_argument("--x-fmt", default="e4m3", choices=["e4m3", "e5m2"],
                    help="activation code format (e5m2: the pages' activation-format variant)")
    ap.add_argument("--weight-scales", default="channel", choices=["channel", "tensor", "block"],
                    help="weight scale granularity: channel (the path), tensor (the pages' FFN variant, dense "
                         "workloads) or block (128x128, the pages' MoE variant, moe workload)")
    ap.add_argument("--fused", action="store_true",
                    help="one fused quantize+linear launch per step where it applies (<= 16 rows); "
                         "default: the two launches, measured faster on B200")
    ap.add_argument("--overlap", action="store_true",
                    help="M > 128: one launch per step that quantizes inside the CTA-pair GEMM")
    ap.add_argument("--gemm", default="auto", choices=["auto", "single", "pair", "splitk"],
                    help="dense GEMM kernel family (tuning sweeps; default: chosen per shape)")
    ap.add_argument("--bn", type=int, default=0, help="pair-kernel tile width (0 = automatic)")
    ap.add_argument("--ksplit", type=int, default=0, help="split-K cluster size for M <= 128 (0 = automatic)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        # host-only arm: rank 0 runs the oracle, other ranks exit without work
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    world, rank, local = dist_setup(args.gpus)
    if True:
        out = run_ours(args, world, rank, local)
        if rank == 0 and out is not None:
            if world == 1 and not args.no_cpu_baseline:
                _, kind, tensors = workload_spec(args.workload)
                out["cpu_baseline"] = cpu_baseline(kind, tensors, x_fmt=args.x_fmt, weights=args.weight_scales)
            else:
                out["cpu_baseline"] = None
    if rank == 0 and out is not None:
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
