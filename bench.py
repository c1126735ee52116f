#!/usr/bin/env python
"""Benchmark of the FP8 scaled-GEMM hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
dynamic quantization of both operands (amax -> scale -> e4m3 cast) and the
scaled GEMM with its epilogue (scales, bias, bf16 cast) -- or, for the MoE
workload, the grouped GEMM over the offs array.  Inputs are resident in HBM
when the timed region starts; L2 is flushed (a 256 MB write) between steps,
outside the per-step CUDA events (and read back, so that L2 holds clean lines).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

Prints ONE JSON line (rank 0).  `value` is GEMM TFLOP/s over the whole step
(quantize + GEMM) summed over ranks; `roofline` describes the GEMM kernel
alone against the measured peak; `e2e` is the same metric through the public
API with host buffers and the copies inside the timed region;
`cpu_baseline` is the CPU oracle on a bounded sample of the same workload.

With --impl reference the oracle itself is timed on the host cores (rank 0
only), as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fp8_scaled_matrix_b200 import workloads as W  # noqa: E402

WORKLOADS = {
    # name: (workload index, shape index)
    "tensorwise_256": (0, 0),
    "rowwise_4096": (1, 0),
    "blockwise_1x128_128x128": (2, 0),
    "blockwise_1x128_128x128_b": (2, 1),
    "blockwise_1x128_128x1": (3, 0),
    "blockwise_1x128_128x1_b": (3, 1),
    "grouped_e16": (4, 0),
    "grad_input_1x128_128x128": (5, 0),
    "grad_weight_1x128_128x1": (6, 0),
    "grouped_e16_blockwise": (7, 0),
    "linear_chain_1x128_128x128": (8, 0),
    "mxfp8_16640x5120x8192": (9, 0),
    "mxfp8_16640x8192x5120": (9, 1),
    "linear_chain_mxfp8": (10, 0),
    "grouped_e16_mxfp8": (11, 0),
    "grouped_e16_grad_input": (12, 0),
    "grouped_e16_grad_weight": (13, 0),
    "linear_chain_train_1x128": (14, 0),
}
DEFAULT_WORKLOAD = "rowwise_4096"
# Page 5's context numbers (TFLOP/s of torch._scaled_mm, hardware not stated)
PAGE_NUMBERS = {
    "blockwise_1x128_128x128": 1008.91, "blockwise_1x128_128x128_b": 1002.23,
    "blockwise_1x128_128x1": 808.271, "blockwise_1x128_128x1_b": 807.015,
}
OPERAND_GROUPS = {"tensor": ("tensor", "tensor"), "row": ("row", "row"),
                  "1x128_128x128": ("1x128", "128x128"),
                  "1x128_128x1": ("1x128", "1x128"), "grouped": ("row", "row"),
                  "grad_input": ("1x128", "128x128"), "grad_weight": ("1x128", "1x128"),
                  "grouped_blockwise": ("1x128", "128x128"), "chain": ("1x128", "128x128"),
                  "mxfp8": ("mx", "mx"), "chain_mx": ("mx", "mx"), "grouped_mx": ("mx", "mx"),
                  "grouped_grad_input": ("1x128", "128x128"),
                  "grouped_grad_weight": ("1x128", "1x128"),
                  "chain_train": ("1x128", "128x128")}
# GEMM recipe of each workload recipe, and which operands are quantized
# transposed (the training GEMMs contract along the stored rows)
GEMM_RECIPE = {"grad_input": "1x128_128x128", "grad_weight": "1x128_128x1",
               "chain": "1x128_128x128"}
TRANSPOSED = {"grad_input": (False, True), "grad_weight": (True, True)}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0   # nominal dense ratio (4.5 / 2.25 PFLOP/s)
L2_FLUSH_BYTES = 256 << 20


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ------------------------------------------------------------------ peaks

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# the GEMM kernel's sources: its recorded DRAM traffic stays valid while
# these are unchanged
GEMM_SOURCES = ("gemm.cu", "sm100.cuh", "status.cuh")


def kernel_sources_hash(files=None) -> str:
    """Hash of the kernel sources (all of csrc/, or the named files)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "fp8_scaled_matrix_b200", "csrc")
    for f in sorted(files if files is not None else os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per GEMM launch from the committed ncu summary, if it was
    taken on the current GEMM kernel sources; otherwise None."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d.get(workload)
        if e and e.get("sources") == kernel_sources_hash(GEMM_SOURCES):
            return float(e["bytes_per_launch"])
    except Exception:
        return None
    return None


# ------------------------------------------------------- multi-rank plumbing

def max_over_ranks(x: float, dev) -> float:
    """The largest of every rank's `x` (a device time): one all-reduce(MAX)
    over the default process group, or `x` itself on a single rank."""
    dist = torch.distributed
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput: every rank's work over the slowest rank's time."""
    return flops_per_rank * world / (ms * 1e-3) / 1e12


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- our path

class Step:
    """Device buffers and the launches of one step of a workload."""

    def __init__(self, wl: W.Workload, dev: torch.device):
        from fp8_scaled_matrix_b200 import fp8sm
        self.f = fp8sm
        self.wl = wl
        self.dev = dev
        ga, gb = OPERAND_GROUPS[wl.recipe]
        self.mx = wl.recipe in ("mxfp8", "chain_mx", "grouped_mx")
        self.qa_recipe = None if self.mx else fp8sm.QUANT_RECIPES[ga]
        self.qb_recipe = None if self.mx else fp8sm.QUANT_RECIPES[gb]
        self.a = wl.a.to(dev)
        self.grouped = wl.recipe in ("grouped", "grouped_blockwise", "grouped_mx",
                                     "grouped_grad_input")
        self.gin = wl.recipe == "grouped_grad_input"
        self.wg = wl.recipe == "grouped_grad_weight"
        if self.wg:
            # (tokens x out) and (tokens x in), quantized per expert, transposed
            self.grouped = False
            self.b = wl.b.to(dev)
            self.offs = wl.offs.to(dev)
        elif self.gin:
            # the experts as stored (E, out, in); each is quantized transposed
            self.b = wl.b.to(dev)
            self.offs = wl.offs.to(dev)
        elif self.grouped:
            E, N, K = wl.b.shape
            self.b = wl.b.to(dev).reshape(E * N, K)
            self.offs = wl.offs.to(dev)
        else:
            self.b = wl.b.to(dev)
            self.offs = None
        self.bias = None if wl.bias is None else wl.bias.to(dev)
        self.t_a, self.t_b = TRANSPOSED.get(wl.recipe, (False, False))
        # quantized operands: A (M, K), B (N, K) (grouped: (E N, K))
        rows_a, rows_b = wl.M, self.b.shape[1] if self.t_b else self.b.shape[0]
        if self.gin:
            rows_b = wl.b.shape[0] * wl.N    # (E * in, out) codes
        cols = wl.K
        if self.wg:
            # per-expert padded transposed operands: (out, P), (in, P)
            rows_a, rows_b = wl.M, wl.N
            cols = fp8sm.fp8_grouped_padded_tokens(wl.K, wl.E)
        self.qa = torch.empty(rows_a, cols, dtype=torch.uint8, device=dev)
        self.qb = torch.empty(rows_b, cols, dtype=torch.uint8, device=dev)
        if self.wg:
            self.sa = torch.empty(cols // 128, rows_a, dtype=torch.float32, device=dev)
            self.sb = torch.empty(cols // 128, rows_b, dtype=torch.float32, device=dev)
        elif self.mx:
            # E8M0 scale-factor tiles
            self.sa = torch.empty(fp8sm.fp8_mx_scale_bytes(rows_a, cols), dtype=torch.uint8,
                                  device=dev)
            self.sb = torch.empty(fp8sm.fp8_mx_scale_bytes(rows_b, cols), dtype=torch.uint8,
                                  device=dev)
        else:
            self.sa = torch.empty(max(fp8sm.scale_count(rows_a, cols, self.qa_recipe), 1),
                                  dtype=torch.float32, device=dev)
            self.sb = torch.empty(max(fp8sm.scale_count(rows_b, cols, self.qb_recipe), 1),
                                  dtype=torch.float32, device=dev)
        self.ws = torch.zeros(64, dtype=torch.uint8, device=dev)
        self.ws_b = torch.zeros(64, dtype=torch.uint8, device=dev)
        self.side = torch.cuda.Stream(device=dev)
        self.ev_fork = torch.cuda.Event()
        self.ev_join = torch.cuda.Event()
        self.out = torch.empty(((wl.E,) if self.wg else ()) + (wl.M, wl.N),
                               dtype=torch.bfloat16, device=dev)
        self.launches_per_step = 3
        if wl.recipe == "grouped_blockwise":
            # each expert's weights are quantized on their own (its 128x128
            # tiles and scales), into the (E, K/128, N/128) scale layout
            E, N, K = wl.b.shape
            self.sb = torch.empty(E * fp8sm.scale_count(N, K, self.qb_recipe),
                                  dtype=torch.float32, device=dev)
        if self.gin:
            # per expert W_g^T quantized 128x128: (out/128, in/128) scales each
            E = wl.b.shape[0]
            self.sb = torch.empty(E * fp8sm.scale_count(wl.N, wl.K, self.qb_recipe),
                                  dtype=torch.float32, device=dev)
        self.chain = wl.recipe in ("chain", "chain_mx")
        if self.chain:
            # second linear: its weight (N2, N) quantized 128x128 like b; the
            # first GEMM's output leaves as e4m3 codes + 1x128 scales
            # ((N/128, M), the A-operand scale layout of the second GEMM)
            self.b2 = wl.extra["b2"].to(dev)
            n2 = self.b2.shape[0]
            self.qb2 = torch.empty(n2, wl.N, dtype=torch.uint8, device=dev)
            self.y1q = torch.empty(wl.M, wl.N, dtype=torch.uint8, device=dev)
            if self.mx:
                self.sb2 = torch.empty(fp8sm.fp8_mx_scale_bytes(n2, wl.N), dtype=torch.uint8,
                                       device=dev)
                self.y1s = torch.empty(fp8sm.fp8_mx_scale_bytes(wl.M, wl.N), dtype=torch.uint8,
                                       device=dev)
            else:
                self.sb2 = torch.empty(fp8sm.scale_count(n2, wl.N, self.qb_recipe),
                                       dtype=torch.float32, device=dev)
                self.y1s = torch.empty(wl.N // 128, wl.M, dtype=torch.float32, device=dev)
            self.out = torch.empty(wl.M, n2, dtype=torch.bfloat16, device=dev)
            self.launches_per_step = 5

    def inputs(self):
        """The device tensors a step reads, in host_inputs' order."""
        t = [self.a, self.b]
        if self.bias is not None:
            t.append(self.bias)
        if self.chain:
            t.append(self.b2)
        return t

    def host_inputs(self):
        """The workload's host tensors in the layout of inputs()."""
        wl = self.wl
        hb = (wl.b.reshape(-1, wl.K)
              if wl.recipe in ("grouped", "grouped_blockwise", "grouped_mx") else wl.b)
        t = [wl.a, hb]
        if wl.bias is not None:
            t.append(wl.bias)
        if self.chain:
            t.append(wl.extra["b2"])
        return t

    def outputs(self):
        return [self.out]

    def quantize(self):
        """Both operands' quantization; the second runs on a side stream,
        concurrently with the first (same work, overlapped), and the main
        stream waits for it before the GEMM."""
        f = self.f
        main = torch.cuda.current_stream()
        self.ev_fork.record(main)
        self.side.wait_event(self.ev_fork)
        with torch.cuda.stream(self.side):
            if self.wg:
                f.fp8_quantize_transposed_grouped(self.b, self.offs, out=self.qb, scales=self.sb,
                                                  stream=self.side)
            elif self.gin:
                # every expert's W_g^T, one launch
                f.fp8_quantize_transposed_batched(self.b, self.qb_recipe, out=self.qb,
                                                  scales=self.sb, stream=self.side)
            elif self.wl.recipe == "grouped_blockwise":
                # every expert's 128x128 tiles and scales, one launch
                E, N, K = self.wl.b.shape
                f.fp8_quantize_batched(self.b.view(E, N, K), self.qb_recipe, out=self.qb,
                                       scales=self.sb, stream=self.side)
            elif self.t_b:
                f.fp8_quantize_transposed(self.b, self.qb_recipe, out=self.qb, scales=self.sb,
                                          stream=self.side)
            elif self.mx:
                f.fp8_quantize_mx(self.b, out=self.qb, scales=self.sb, stream=self.side)
                if self.chain:
                    f.fp8_quantize_mx(self.b2, out=self.qb2, scales=self.sb2, stream=self.side)
            elif self.chain:
                f.fp8_quantize(self.b, self.qb_recipe, out=self.qb, scales=self.sb,
                               workspace=self.ws_b, stream=self.side)
                f.fp8_quantize(self.b2, self.qb_recipe, out=self.qb2, scales=self.sb2,
                               workspace=self.ws_b, stream=self.side)
            else:
                f.fp8_quantize(self.b, self.qb_recipe, out=self.qb, scales=self.sb,
                               workspace=self.ws_b, stream=self.side)
        if self.wg:
            f.fp8_quantize_transposed_grouped(self.a, self.offs, out=self.qa, scales=self.sa,
                                              stream=main)
        elif self.mx:
            f.fp8_quantize_mx(self.a, out=self.qa, scales=self.sa, stream=main)
        elif self.t_a:
            f.fp8_quantize_transposed(self.a, self.qa_recipe, out=self.qa, scales=self.sa,
                                      stream=main)
        else:
            f.fp8_quantize(self.a, self.qa_recipe, out=self.qa, scales=self.sa,
                           workspace=self.ws, stream=main)
        self.ev_join.record(self.side)
        main.wait_event(self.ev_join)

    def gemm(self):
        f = self.f
        wl = self.wl
        if wl.recipe == "grouped":
            E, N, K = wl.b.shape
            f.fp8_grouped_scaled_mm(self.qa, self.qb.view(E, N, K), self.sa,
                                    self.sb.view(E, N), self.offs, out=self.out)
        elif wl.recipe == "grouped_blockwise":
            E, N, K = wl.b.shape
            f.fp8_grouped_scaled_mm_blockwise(self.qa, self.qb.view(E, N, K), self.sa,
                                              self.sb, self.offs, out=self.out)
        elif self.wg:
            f.fp8_grouped_scaled_mm_wgrad(self.qa, self.qb, self.sa, self.sb, self.offs, wl.K,
                                          out=self.out)
        elif self.gin:
            E = wl.b.shape[0]
            f.fp8_grouped_scaled_mm_blockwise(self.qa, self.qb.view(E, wl.N, wl.K), self.sa,
                                              self.sb, self.offs, out=self.out)
        elif wl.recipe == "grouped_mx":
            E, N, K = wl.b.shape
            f.fp8_grouped_scaled_mm_mx(self.qa, self.qb.view(E, N, K), self.sa, self.sb,
                                       self.offs, out=self.out)
        elif self.mx and self.chain:
            f.fp8_scaled_mm_mx_quantized(self.qa, self.qb, self.sa, self.sb,
                                         out=self.y1q, out_scales=self.y1s)
            f.fp8_scaled_mm_mx(self.y1q, self.qb2, self.y1s, self.sb2, out=self.out)
        elif self.mx:
            f.fp8_scaled_mm_mx(self.qa, self.qb, self.sa, self.sb, bias=self.bias, out=self.out)
        elif self.chain:
            r = f.MM_RECIPES["1x128_128x128"]
            f.fp8_scaled_mm_quantized(self.qa, self.qb, self.sa, self.sb, r,
                                      out=self.y1q, out_scales=self.y1s)
            f.fp8_scaled_mm(self.y1q, self.qb2, self.y1s, self.sb2, r, out=self.out)
        else:
            f.fp8_scaled_mm(self.qa, self.qb, self.sa, self.sb,
                            f.MM_RECIPES[GEMM_RECIPE.get(wl.recipe, wl.recipe)],
                            bias=self.bias, out=self.out)

    def quant_bytes(self) -> int:
        """Algorithmic HBM bytes of the two quantize launches: 2 B read +
        1 B written per element, 4 B per scale."""
        n = self.a.numel() + self.b.numel()
        b = 3 * n + self.sa.element_size() * self.sa.numel() + \
            self.sb.element_size() * self.sb.numel()
        if self.chain:
            b += 3 * self.b2.numel() + self.sb2.element_size() * self.sb2.numel()
        return b


class TrainStep:
    """Forward and backward of the two-linear chain X -> W1 -> W2, blockwise
    scaled throughout ("improve fp8 blockwise gemm perf": 1x128_128x128 for
    the forward and grad_input GEMMs, 1x128_128x1 for grad_weight).

    quantize(): X and dY2 in 1x128 groups along the features and, transposed,
    along the tokens; W1 and W2 in 128x128 tiles, as stored and transposed.
    gemm(): Y1 = X W1^T and dY1 = dY2 W2 write both e4m3 forms of their
    result from the epilogue; Y2 = Y1 W2^T, dX = dY1 W1, dW1 = dY1^T X and
    dW2 = dY2^T Y1 read them.  All outputs bf16."""

    def __init__(self, wl: W.Workload, dev: torch.device):
        from fp8_scaled_matrix_b200 import fp8sm
        self.f = fp8sm
        self.wl = wl
        T, F, D = wl.M, wl.N, wl.K
        self.x, self.w1 = wl.a.to(dev), wl.b.to(dev)
        self.w2, self.dy2 = wl.extra["b2"].to(dev), wl.extra["dy"].to(dev)

        def u8(r, c):
            return torch.empty(r, c, dtype=torch.uint8, device=dev)

        def f32(r, c):
            return torch.empty(r, c, dtype=torch.float32, device=dev)

        def bf(r, c):
            return torch.empty(r, c, dtype=torch.bfloat16, device=dev)
        # activations: 1x128 scales (cols/128, rows); weights: 128x128 scales
        # (cols/128, rows/128)
        self.qx, self.sx, self.qxt, self.sxt = u8(T, D), f32(D // 128, T), u8(D, T), f32(T // 128, D)
        self.qd, self.sd, self.qdt, self.sdt = u8(T, D), f32(D // 128, T), u8(D, T), f32(T // 128, D)
        self.qw1, self.sw1 = u8(F, D), f32(D // 128, F // 128)
        self.qw1t, self.sw1t = u8(D, F), f32(F // 128, D // 128)
        self.qw2, self.sw2 = u8(D, F), f32(F // 128, D // 128)
        self.qw2t, self.sw2t = u8(F, D), f32(D // 128, F // 128)
        self.y1 = (u8(T, F), f32(F // 128, T), u8(F, T), f32(T // 128, F))
        self.dy1 = (u8(T, F), f32(F // 128, T), u8(F, T), f32(T // 128, F))
        self.y2, self.dx, self.dw1, self.dw2 = bf(T, D), bf(T, D), bf(F, D), bf(D, F)
        self.side = torch.cuda.Stream(device=dev)
        self.ev_fork = torch.cuda.Event()
        self.ev_join = torch.cuda.Event()
        self.launches_per_step = 14

    def inputs(self):
        return [self.x, self.w1, self.w2, self.dy2]

    def host_inputs(self):
        wl = self.wl
        return [wl.a, wl.b, wl.extra["b2"], wl.extra["dy"]]

    def outputs(self):
        return [self.y2, self.dx, self.dw1, self.dw2]

    def quantize(self):
        f = self.f
        B1, B128 = f.FP8_SCALE_BLOCK_1x128, f.FP8_SCALE_BLOCK_128x128
        main = torch.cuda.current_stream()
        self.ev_fork.record(main)
        self.side.wait_event(self.ev_fork)
        with torch.cuda.stream(self.side):
            f.fp8_quantize(self.w1, B128, out=self.qw1, scales=self.sw1, stream=self.side)
            f.fp8_quantize(self.w2, B128, out=self.qw2, scales=self.sw2, stream=self.side)
            f.fp8_quantize_transposed(self.w1, B128, out=self.qw1t, scales=self.sw1t,
                                      stream=self.side)
            f.fp8_quantize_transposed(self.w2, B128, out=self.qw2t, scales=self.sw2t,
                                      stream=self.side)
        f.fp8_quantize(self.x, B1, out=self.qx, scales=self.sx, stream=main)
        f.fp8_quantize_transposed(self.x, B1, out=self.qxt, scales=self.sxt, stream=main)
        f.fp8_quantize(self.dy2, B1, out=self.qd, scales=self.sd, stream=main)
        f.fp8_quantize_transposed(self.dy2, B1, out=self.qdt, scales=self.sdt, stream=main)
        self.ev_join.record(self.side)
        main.wait_event(self.ev_join)

    def gemm(self):
        f = self.f
        R, R1 = f.FP8_MM_1x128_128x128, f.FP8_MM_1x128_128x1
        y1q, y1s, y1tq, y1ts = self.y1
        d1q, d1s, d1tq, d1ts = self.dy1
        f.fp8_scaled_mm_quantized_dual(self.qx, self.qw1, self.sx, self.sw1, R, out=y1q,
                                       out_scales=y1s, out_t=y1tq, out_t_scales=y1ts)
        f.fp8_scaled_mm(y1q, self.qw2, y1s, self.sw2, R, out=self.y2)
        f.fp8_scaled_mm_quantized_dual(self.qd, self.qw2t, self.sd, self.sw2t, R, out=d1q,
                                       out_scales=d1s, out_t=d1tq, out_t_scales=d1ts)
        f.fp8_scaled_mm(d1q, self.qw1t, d1s, self.sw1t, R, out=self.dx)
        f.fp8_scaled_mm(d1tq, self.qxt, d1ts, self.sxt, R1, out=self.dw1)
        f.fp8_scaled_mm(self.qdt, y1tq, self.sdt, y1ts, R1, out=self.dw2)

    def quant_bytes(self) -> int:
        """Algorithmic HBM bytes of the eight quantize launches: 2 B read +
        1 B written per element, 4 B per scale."""
        act = self.x.numel() + self.dy2.numel()
        w = self.w1.numel() + self.w2.numel()
        sc = sum(t.numel() * 4 for t in (self.sx, self.sxt, self.sd, self.sdt, self.sw1,
                                         self.sw1t, self.sw2, self.sw2t))
        return 2 * 3 * (act + w) + sc


def make_step(wl: W.Workload, dev: torch.device):
    return TrainStep(wl, dev) if wl.recipe == "chain_train" else Step(wl, dev)


def evict_l2(flush: torch.Tensor):
    """Write a buffer twice the size of L2, then read it back: the step's
    inputs leave L2, and the lines left behind are clean, so the next kernel
    does not pay for writing the flush buffer back to HBM."""
    flush.zero_()
    flush.sum()


def capture(fn, pool=None):
    """Record the launches `fn` makes (through the C ABI) into a CUDA graph."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, pool=pool):
        fn()
    return g


def run_ours(args, wl, dev, rank, world):
    torch.cuda.set_device(dev)
    st = make_step(wl, dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        st.quantize()
        st.gemm()
    torch.cuda.synchronize()
    st.f.check_device_status()
    quantize, gemm = st.quantize, st.gemm
    if args.graphs:
        # The step's launches replayed from CUDA graphs: the same kernels on
        # the same buffers, without the host's per-call cost between them.
        gq = capture(st.quantize)
        gg = capture(st.gemm, pool=gq.pool())
        quantize, gemm = gq.replay, gg.replay
        for _ in range(3):
            quantize()
            gemm()
        torch.cuda.synchronize()
        st.f.check_device_status()
    stream = torch.cuda.current_stream()

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.25)  # let the sampler start before the timed work
    for i in range(K):
        evict_l2(flush)  # outside the step's events
        ev[i][0].record(stream)
        quantize()
        ev[i][1].record(stream)
        gemm()
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    st.f.check_device_status()
    q_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    g_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(K)]
    step_ms = [q + g for q, g in zip(q_ms, g_ms)]
    total_ms = max_over_ranks(float(np.sum(step_ms)), dev)
    res = {
        "total_ms": total_ms,
        "q_ms": float(np.mean(q_ms)), "g_ms": float(np.mean(g_ms)),
        "g_ms_median": float(np.median(g_ms)), "q_ms_median": float(np.median(q_ms)),
        "quant_bytes": st.quant_bytes(), "launches": st.launches_per_step * K,
        "clocks": clocks,
    }
    if not args.no_e2e:
        res["e2e"] = run_e2e(args, wl, dev, world)
    return res


def run_e2e(args, wl, dev, world):
    """Same step through the public API from pinned HOST buffers: every step
    copies its bf16 inputs host -> device, quantizes, multiplies, and copies
    its results device -> host, all inside the timed region.  Steps are
    pipelined the way a serving loop would run them: two sets of device
    buffers and three streams (upload, compute, download), so step i's
    download and step i+1's upload overlap each other and the compute; every
    copy of every step is still made and timed."""
    from fp8_scaled_matrix_b200 import fp8sm  # noqa: F401
    sets = [make_step(wl, dev), make_step(wl, dev)]
    hin = [t.contiguous().pin_memory() for t in sets[0].host_inputs()]
    hout = [[torch.empty(tuple(o.shape), dtype=o.dtype).pin_memory()
             for o in sets[0].outputs()] for _ in range(2)]
    s_in, s_comp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    steps = max(3, min(args.steps, args.e2e_steps))

    def one(i):
        k = i % 2
        st = sets[k]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_comp[k])   # step i-2 has consumed set k's inputs
            for d, h in zip(st.inputs(), hin):
                d.copy_(h, non_blocking=True)
            ev_in[k].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[k])
            if i >= 2:
                s_comp.wait_event(ev_out[k])  # step i-2's results have left set k
            st.quantize()
            st.gemm()
            ev_comp[k].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[k])
            for h, d in zip(hout[k], st.outputs()):
                h.copy_(d, non_blocking=True)
            ev_out[k].record(s_out)

    for i in range(2):
        one(i)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        one(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_comp)
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, dev)
    h2d = sum(t.numel() * t.element_size() for t in hin)
    d2h = sum(t.numel() * t.element_size() for t in hout[0])
    return {"ms": ms, "h2d": h2d, "d2h": d2h, "steps": steps}


# ---------------------------------------------------------------- oracle

def oracle_sample(wl, max_rows: int):
    """Time the CPU oracle on a bounded sample of the workload: quantize of
    both operands in full, the GEMM on the first `max_rows` output rows.
    Returns (seconds for the sample, fraction of the GEMM it covers,
    seconds for quantize, threads)."""
    import oracle
    ga, gb = OPERAND_GROUPS[wl.recipe]
    G = {"tensor": oracle.GROUP_TENSOR, "row": oracle.GROUP_ROW,
         "1x128": oracle.GROUP_1x128, "128x128": oracle.GROUP_128x128}
    MMR = {"tensor": oracle.MM_TENSOR_TENSOR, "row": oracle.MM_ROW_ROW,
           "1x128_128x128": oracle.MM_1x128_128x128, "1x128_128x1": oracle.MM_1x128_128x1}
    t_a, t_b = TRANSPOSED.get(wl.recipe, (False, False))

    def bits(x, transposed):
        b = W.bf16_bits(x)
        return np.ascontiguousarray(b.T) if transposed else b
    t0 = time.perf_counter()
    if wl.recipe == "chain_train":
        # the whole step on the first tokens (a multiple of 128, the length of
        # the transposed groups): each of the six GEMMs and the activation
        # quantizes cost in proportion to the token count; the weights'
        # quantization (as stored and transposed) is timed in full
        G1, G128 = oracle.GROUP_1x128, oracle.GROUP_128x128
        R, R1 = MMR["1x128_128x128"], MMR["1x128_128x1"]
        w1b, w2b = W.bf16_bits(wl.b), W.bf16_bits(wl.extra["b2"])
        qw1, sw1 = oracle.quantize(w1b, G128)
        qw2, sw2 = oracle.quantize(w2b, G128)
        qw1t, sw1t = oracle.quantize(np.ascontiguousarray(w1b.T), G128)
        qw2t, sw2t = oracle.quantize(np.ascontiguousarray(w2b.T), G128)
        tq = time.perf_counter() - t0
        t = min(wl.M, -(-max(1, max_rows) // 128) * 128)
        t0 = time.perf_counter()
        xb, db = W.bf16_bits(wl.a[:t]), W.bf16_bits(wl.extra["dy"][:t])
        qx, sx = oracle.quantize(xb, G1)
        qxt, sxt = oracle.quantize(np.ascontiguousarray(xb.T), G1)
        qd, sd = oracle.quantize(db, G1)
        qdt, sdt = oracle.quantize(np.ascontiguousarray(db.T), G1)
        y1 = oracle.scaled_mm(qx, qw1, sx, sw1, R)[0].astype(np.float32)
        y1q, y1s = oracle.quantize_f32(y1, G1)
        y1tq, y1ts = oracle.quantize_f32(np.ascontiguousarray(y1.T), G1)
        oracle.scaled_mm(y1q, qw2, y1s, sw2, R)
        dy1 = oracle.scaled_mm(qd, qw2t, sd, sw2t, R)[0].astype(np.float32)
        d1q, d1s = oracle.quantize_f32(dy1, G1)
        d1tq, d1ts = oracle.quantize_f32(np.ascontiguousarray(dy1.T), G1)
        oracle.scaled_mm(d1q, qw1t, d1s, sw1t, R)
        oracle.scaled_mm(d1tq, qxt, d1ts, sxt, R1)
        oracle.scaled_mm(qdt, y1tq, sdt, y1ts, R1)
        return time.perf_counter() - t0, t / wl.M, tq, oracle.num_threads()
    if wl.recipe == "chain_mx":
        qa, sa = oracle.mx_quantize(W.bf16_bits(wl.a))
        qb, sb = oracle.mx_quantize(W.bf16_bits(wl.b))
        qb2, sb2 = oracle.mx_quantize(W.bf16_bits(wl.extra["b2"]))
        tq = time.perf_counter() - t0
        rows = np.arange(min(max_rows, wl.M), dtype=np.int64)
        t0 = time.perf_counter()
        y1, _ = oracle.mx_scaled_mm(qa, qb, sa, sb, rows=rows)
        y1q, y1e = oracle.mx_quantize_f32(y1.astype(np.float32))
        oracle.mx_scaled_mm(y1q, qb2, y1e, sb2)
        return time.perf_counter() - t0, rows.size / wl.M, tq, oracle.num_threads()
    if wl.recipe == "mxfp8":
        qa, sa = oracle.mx_quantize(W.bf16_bits(wl.a))
        qb, sb = oracle.mx_quantize(W.bf16_bits(wl.b))
        tq = time.perf_counter() - t0
        rows = np.arange(min(max_rows, wl.M), dtype=np.int64)
        t0 = time.perf_counter()
        oracle.mx_scaled_mm(qa, qb, sa, sb, rows=rows)
        return time.perf_counter() - t0, rows.size / wl.M, tq, oracle.num_threads()
    if wl.recipe == "grouped_grad_weight":
        # each expert's zero-padded transposed slices, quantized 1x128; the
        # GEMM on the first max_rows output rows of every expert
        ends = wl.offs.numpy()
        ops = []
        start = 0
        for end in ends:
            n = int(end) - start
            if n:
                pad = -(-n // 128) * 128
                ta = np.zeros((wl.M, pad), np.uint16)
                tb = np.zeros((wl.N, pad), np.uint16)
                ta[:, :n] = W.bf16_bits(wl.a[start:int(end)]).T
                tb[:, :n] = W.bf16_bits(wl.b[start:int(end)]).T
                ops.append(oracle.quantize(ta, G["1x128"]) + oracle.quantize(tb, G["1x128"]))
            start = int(end)
        tq = time.perf_counter() - t0
        rows = np.arange(min(max_rows, wl.M), dtype=np.int64)
        t0 = time.perf_counter()
        for qa, sa, qb, sb in ops:
            oracle.scaled_mm(qa, qb, sa, sb, MMR["1x128_128x1"], rows=rows)
        return time.perf_counter() - t0, rows.size / wl.M, tq, oracle.num_threads()
    if wl.recipe == "grouped_grad_input":
        qa, sa = oracle.quantize(W.bf16_bits(wl.a), G["1x128"])
        per_expert = [oracle.quantize(np.ascontiguousarray(W.bf16_bits(wl.b[e]).T), G["128x128"])
                      for e in range(wl.b.shape[0])]
        tq = time.perf_counter() - t0
        rows = np.arange(min(max_rows, wl.M), dtype=np.int64)
        t0 = time.perf_counter()
        sa2 = sa.reshape(wl.K // 128, wl.M)
        start = 0
        for e, end in enumerate(wl.offs.numpy()):
            sel = rows[(rows >= start) & (rows < end)]
            if sel.size:
                oracle.scaled_mm(np.ascontiguousarray(qa[start:end]), per_expert[e][0],
                                 np.ascontiguousarray(sa2[:, start:end]).reshape(-1),
                                 per_expert[e][1], MMR["1x128_128x128"], rows=sel - start)
            start = int(end)
        return time.perf_counter() - t0, rows.size / wl.M, tq, oracle.num_threads()
    if wl.recipe == "grouped_mx":
        E, N, K = wl.b.shape
        qa, sa = oracle.mx_quantize(W.bf16_bits(wl.a))
        qb, sb = oracle.mx_quantize(W.bf16_bits(wl.b.reshape(E * N, K)))
        tq = time.perf_counter() - t0
        rows = np.arange(min(max_rows, wl.M), dtype=np.int64)
        t0 = time.perf_counter()
        start = 0
        for e, end in enumerate(wl.offs.numpy()):
            sel = rows[(rows >= start) & (rows < end)]
            if sel.size:
                oracle.mx_scaled_mm(np.ascontiguousarray(qa[start:end]), qb[e * N:(e + 1) * N],
                                    np.ascontiguousarray(sa[start:end]), sb[e * N:(e + 1) * N],
                                    rows=sel - start)
            start = int(end)
        return time.perf_counter() - t0, rows.size / wl.M, tq, oracle.num_threads()
    qa, sa = oracle.quantize(bits(wl.a, t_a), G[ga])
    if wl.recipe == "grouped":
        E, N, K = wl.b.shape
        qb, sb = oracle.quantize(W.bf16_bits(wl.b.reshape(E * N, K)), G[gb])
    elif wl.recipe == "grouped_blockwise":
        per_expert = [oracle.quantize(W.bf16_bits(wl.b[e].contiguous()), G[gb])
                      for e in range(wl.b.shape[0])]
        qb = np.stack([q for q, _ in per_expert])
        sb = np.stack([s for _, s in per_expert])
    else:
        qb, sb = oracle.quantize(bits(wl.b, t_b), G[gb])
    if wl.recipe == "chain":
        qb2, sb2 = oracle.quantize(W.bf16_bits(wl.extra["b2"]), G[gb])
    tq = time.perf_counter() - t0
    rows = np.arange(min(max_rows, wl.M), dtype=np.int64)
    t0 = time.perf_counter()
    if wl.recipe == "grouped":
        E, N, K = wl.b.shape
        oracle.grouped_scaled_mm(qa, qb.reshape(E, N, K), sa, sb.reshape(E, N),
                                 wl.offs.numpy(), rows=rows)
    elif wl.recipe == "grouped_blockwise":
        # the dense blockwise GEMM of each group that the sampled rows touch
        KB = wl.K // 128
        sa2 = sa.reshape(KB, wl.M)
        start = 0
        for e, end in enumerate(wl.offs.numpy()):
            sel = rows[(rows >= start) & (rows < end)]
            if sel.size:
                oracle.scaled_mm(np.ascontiguousarray(qa[start:end]), qb[e],
                                 np.ascontiguousarray(sa2[:, start:end]).reshape(-1),
                                 sb[e].reshape(-1), MMR["1x128_128x128"], rows=sel - start)
            start = int(end)
    elif wl.recipe == "chain":
        # first linear on the sampled rows, its fp32 result quantized 1x128,
        # then the second linear on those rows
        y1, _ = oracle.scaled_mm(qa, qb, sa, sb, MMR["1x128_128x128"], rows=rows)
        y1q, y1s = oracle.quantize_f32(y1.astype(np.float32), oracle.GROUP_1x128)
        oracle.scaled_mm(y1q, qb2, y1s, sb2, MMR["1x128_128x128"])
    else:
        bias = None if wl.bias is None else W.bf16_bits(wl.bias)
        oracle.scaled_mm(qa, qb, sa, sb, MMR[GEMM_RECIPE.get(wl.recipe, wl.recipe)],
                         bias_bits=bias, rows=rows)
    tg = time.perf_counter() - t0
    return tg, rows.size / wl.M, tq, oracle.num_threads()


def cpu_baseline(wl, rows: int):
    tg, frac, tq, threads = oracle_sample(wl, rows)
    est_s = tq + tg / frac
    value = wl.flops / est_s / 1e12
    if wl.recipe == "chain_train":
        t = int(round(frac * wl.M))
        return {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                "sample": (f"quantize of W1 and W2, as stored and transposed, in full "
                           f"({tq:.2f} s) + the rest of the step (activation quantizes, six "
                           f"GEMMs, both quantized forms of Y1 and dY1) on the first {t} of "
                           f"{wl.M} tokens ({tg:.2f} s), scaled to all rows"),
                "seconds_est_per_step": est_s}
    chain = wl.recipe in ("chain", "chain_mx")
    what = "X, W1 and W2" if chain else "both operands"
    gemm = (("both GEMMs (the first one's fp32 output quantized "
             + ("MXFP8)" if wl.recipe == "chain_mx" else "1x128)")) if chain else "GEMM")
    return {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": (f"quantize of {what} in full ({tq:.2f} s) + {gemm} on "
                       f"{int(round(frac * wl.M))} of {wl.M} output rows ({tg:.2f} s), "
                       f"scaled to all rows"),
            "seconds_est_per_step": est_s}


def baseline_rows(wl, target_s: float = 12.0) -> int:
    """Rows of the GEMM that take about target_s on the oracle (probe with 8)."""
    tg, frac, _, _ = oracle_sample(wl, 8)
    per_row = tg / max(1, int(round(frac * wl.M)))
    if wl.recipe == "chain_train":   # samples are whole 128-token groups
        return int(max(128, min(wl.M, 128 * round(target_s / max(per_row * 128, 1e-9)))))
    return int(max(8, min(wl.M, target_s / max(per_row, 1e-9))))


# ------------------------------------------------------------------ main

def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--graphs", type=int, default=1, choices=[0, 1],
                    help="replay the step's launches from CUDA graphs (1, default) or "
                         "call the API per launch (0)")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=0,
                    help="output rows for the CPU oracle sample (0: about 12 s of work)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    idx, shape_index = WORKLOADS[args.workload]

    if args.impl == "reference":
        if rank != 0:
            return 0
        wl = W.make_workload(idx, shape_index)
        steps = args.steps or 1
        rows = args.cpu_rows or baseline_rows(wl, 20.0 / max(1, steps + args.warmup))
        for _ in range(min(args.warmup, 1)):
            oracle_sample(wl, max(8, rows // 4))
        times = []
        for _ in range(steps):
            b = cpu_baseline(wl, rows)
            times.append(b["seconds_est_per_step"])
        ms = float(np.mean(times)) * 1e3
        value = wl.flops / (ms * 1e-3) / 1e12
        line = {
            "impl": "reference", "metric": "fp8_scaled_gemm_tflops", "value": value,
            "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp8e4m3/int64-exact/f64", "data": "synthetic",
            "config": {"workload": args.workload, "M": wl.M, "N": wl.N, "K": wl.K},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": b["cores"],
                             "kind": "oracle", "sample": b["sample"]},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return 0

    if world > 1:
        torch.cuda.set_device(local_rank)
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local_rank)
    from fp8_scaled_matrix_b200 import build
    build.build()

    wl = W.make_workload(idx, shape_index)
    if args.steps is None:
        # about a second of timed work per workload
        args.steps = {"tensorwise_256": 4000, "rowwise_4096": 3000,
                      "grouped_e16": 1000}.get(args.workload, 600)
    res = run_ours(args, wl, dev, rank, world)

    peaks, peak_src = load_peaks()
    fp8_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])) * FP8_OVER_BF16
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    K = args.steps
    ms_per_step = res["total_ms"] / K
    value = job_tflops(wl.flops, world, ms_per_step)
    gemm_tflops = wl.flops / (res["g_ms"] * 1e-3) / 1e12
    quant_gbs = res["quant_bytes"] / (res["q_ms"] * 1e-3) / 1e9
    line = {
        "metric": "fp8_scaled_gemm_tflops",
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": (value / world / PAGE_NUMBERS[args.workload]
                        if args.workload in PAGE_NUMBERS else None),
        "dtype": "fp8e4m3 (fp32 accumulate)",
        "data": "synthetic",
        "config": {
            "workload": args.workload, "M": wl.M, "N": wl.N, "K": wl.K,
            "recipe": wl.recipe, "E": wl.E or None, "bias": wl.bias is not None,
            "out_dtype": "bf16",
            "l2": "flushed between steps (256 MB write + read back, outside the step events)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "step": ("quantize X || quantize W1, W2 (two streams), then GEMM1 with its "
                     "output quantized 1x128 in the epilogue, then GEMM2"
                     if wl.recipe == "chain" else
                     "MXFP8 quantize X || W1, W2 (two streams), then GEMM1 with MXFP8 "
                     "output, then GEMM2" if wl.recipe == "chain_mx" else
                     "quantize X, X^T, dY2, dY2^T || W1, W2, W1^T, W2^T (two streams), then "
                     "the chain's forward (Y1 = X W1^T writing Y1 and Y1^T in e4m3, Y2 = Y1 "
                     "W2^T) and backward (dY1 = dY2 W2 writing dY1 and dY1^T in e4m3, dX = "
                     "dY1 W1, dW1 = dY1^T X, dW2 = dY2^T Y1)"
                     if wl.recipe == "chain_train" else
                     "quantize A || quantize B (two streams), then scaled GEMM"),
            "N2": (int(wl.extra["b2"].shape[0]) if "b2" in wl.extra else None),
            "launch": ("CUDA graphs of the step's C-ABI launches" if args.graphs
                       else "one C-ABI call per launch"),
            "e2e": ("pinned host inputs, every step's H2D + quantize + GEMM + D2H of its "
                    "bf16 results; steps pipelined over two buffer sets and three streams"),
        },
        "roofline": {
            "bound": "tensor", "achieved": gemm_tflops, "peak": fp8_peak,
            "unit": "TFLOP/s", "frac": gemm_tflops / fp8_peak,
            "traffic": recorded_traffic(args.workload),
            "kernel": "fp8_gemm_kernel", "peak_source":
                f"{peak_src} bf16 burst x {FP8_OVER_BF16:g} (nominal fp8/bf16 dense ratio)",
            "ms_per_launch": res["g_ms"],
        },
        "roofline_quantize": {
            "bound": "hbm", "achieved": quant_gbs, "peak": hbm_peak, "unit": "GB/s",
            "frac": quant_gbs / hbm_peak, "ms_per_step": res["q_ms"],
            "bytes_per_step": res["quant_bytes"], "peak_source": peak_src,
        },
        "gpu_launches": res["launches"],
        "clocks": res["clocks"],
    }
    if "e2e" in res:
        e = res["e2e"]
        line["e2e"] = {"value": job_tflops(wl.flops, world, e["ms"]), "unit": "TFLOP/s",
                       "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"],
                       "ms_per_step": e["ms"], "steps": e["steps"]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = args.cpu_rows or baseline_rows(wl)
        line["cpu_baseline"] = {k: v for k, v in cpu_baseline(wl, rows).items()
                                if k != "seconds_est_per_step"}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
