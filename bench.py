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

Prints ONE JSON line (rank 0).  The default workload is the blockwise
1x128_128x128 GEMM at M=16640, N=5120, K=8192.  `value` is GEMM TFLOP/s over
the whole step (quantize + GEMM) summed over ranks; `roofline` describes the
GEMM kernel alone against the measured peak (and the nominal one);
`all_configs` times the quantize step and the GEMM of each of the five
benchmark configurations (both (N, K) shapes of the blockwise pair) in the
same process, with the same L2 flush; `e2e` is the same metric through the
public API with host buffers and the copies inside the timed region;
`cpu_baseline` is the CPU oracle on a bounded sample of the same workload;
`clocks` summarises NVML samples taken inside the timed window.

With --impl reference the oracle itself is timed on the host cores (rank 0
only), as the reference arm: every step is the same bounded sample, and the
line reports the time of the steps it ran.
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
# The headline: the blockwise 1x128_128x128 GEMM, M=16640, N=5120, K=8192
# (the first shape of the "improve fp8 blockwise gemm perf" benchmark table)
DEFAULT_WORKLOAD = "blockwise_1x128_128x128"
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
NOMINAL_FP8_TFLOPS = 4500.0   # B200 dense FP8, nominal
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


def rank_shard_rows(a: torch.Tensor, rank: int, world: int) -> torch.Tensor:
    """Data parallel over M (weak scaling): rank r works on its own shard of
    the global batch -- the workload's activation rows rotated by
    r * M / world, same shape and distribution on every rank -- while the
    second operand (the weights) is the same everywhere."""
    return torch.roll(a, shifts=rank * (a.shape[0] // world), dims=0)


def job_tflops(flops_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput: every rank's work over the slowest rank's time."""
    return flops_per_rank * world / (ms * 1e-3) / 1e12


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, read through NVML
    every few milliseconds on a background thread (nvidia-smi's fields,
    sampled fast enough that a timed region of a few milliseconds still gets
    samples).  `window(t0, t1)` summarises the samples taken between two
    host times (time.perf_counter())."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4),
               ("hw_power_brake_slowdown", 0x80))

    def __init__(self, dev: torch.device, interval_s: float = 0.004):
        self.dev = dev
        self.interval = interval_s
        self.samples = []      # (t, sm_mhz, power_w, clock-event reasons bitmask, gpu util %)
        self.max_mhz = None
        self.handle = None
        self.source = None
        self._stop = threading.Event()
        self._t = None

    def _open(self):
        import pynvml
        pynvml.nvmlInit()
        h = None
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            h = pynvml.nvmlDeviceGetHandleByIndex(self.dev.index or 0)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        return pynvml, h

    def start(self):
        try:
            nv, h = self._open()
        except Exception:
            self.source = "unavailable"
            return
        self.source = "nvml"
        getr = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                       getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))

        def run():
            while not self._stop.is_set():
                try:
                    t = time.perf_counter()
                    sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                    rs = int(getr(h)) if getr else 0
                    ut = nv.nvmlDeviceGetUtilizationRates(h).gpu
                    self.samples.append((t, sm, pw, rs, ut))
                except Exception:
                    pass
                self._stop.wait(self.interval)
        self._t = threading.Thread(target=run, daemon=True)
        self._t.start()

    def stop(self):
        self._stop.set()
        if self._t is not None:
            self._t.join(timeout=2)

    GPU_IDLE = 0x1   # NVML clock-event reason: the GPU is idle

    def window(self, t0: float, t1: float) -> dict:
        """Samples taken inside [t0, t1]: median SM clock, the reasons seen
        active, and how many samples fell in the window and under load (the
        driver's GPU-idle clock-event reason not set)."""
        sel = [x for x in self.samples if t0 <= x[0] <= t1]
        load = [x for x in sel if not (x[3] & self.GPU_IDLE)]
        use = load or sel
        reasons = sorted({n for x in use for n, bit in self.REASONS if x[3] & bit})
        return {"sm_mhz": float(np.median([x[1] for x in use])) if use else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(sel), "samples_under_load": len(load),
                "power_w_max": max((x[2] for x in sel), default=None),
                "window_ms": (t1 - t0) * 1e3, "source": self.source}


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
        # both operands on one stream when B takes the 128x128 tile kernel
        # through fp8_quantize (and A the 1x128 kernel)
        self.serial_quant = (wl.recipe in ("1x128_128x128", "chain") and not self.t_a
                             and not self.t_b)
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
        stream waits for it before the GEMM.  When B is quantized in 128x128
        tiles (the TMA-fed tile kernel) both run on the main stream, B's
        first: measured, the tile kernel and the 1x128 kernel run faster one
        after the other than side by side."""
        f = self.f
        main = torch.cuda.current_stream()
        if self.serial_quant:
            f.fp8_quantize(self.b, self.qb_recipe, out=self.qb, scales=self.sb,
                           workspace=self.ws_b, stream=main)
            if self.chain:
                f.fp8_quantize(self.b2, self.qb_recipe, out=self.qb2, scales=self.sb2,
                               workspace=self.ws_b, stream=main)
            f.fp8_quantize(self.a, self.qa_recipe, out=self.qa, scales=self.sa,
                           workspace=self.ws, stream=main)
            return
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


def run_ours(args, wl, dev, rank, world, sampler):
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
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(K):
        evict_l2(flush)  # outside the step's events
        ev[i][0].record(stream)
        quantize()
        ev[i][1].record(stream)
        gemm()
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    if world > 1:
        torch.distributed.barrier()
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
        "clocks": sampler.window(t0, t1),
    }
    del st, flush
    if args.graphs:
        del gq, gg
    torch.cuda.empty_cache()
    if not args.no_e2e:
        res["e2e"] = run_e2e(args, wl, dev, world)
    return res


# The five configurations the benchmark is specified on, as workloads: the
# tensorwise 256^3 GEMM, the rowwise 4096^3 linear, the blockwise
# 1x128_128x128 and 1x128_128x1 GEMMs at both (N, K) shapes of the
# "improve fp8 blockwise gemm perf" tables, and the grouped MoE GEMM.
ALL_CONFIGS = ("tensorwise_256", "rowwise_4096", "blockwise_1x128_128x128",
               "blockwise_1x128_128x128_b", "blockwise_1x128_128x1", "blockwise_1x128_128x1_b",
               "grouped_e16")


def measure_config(name: str, dev, reps: int, fp8_peak: float, hbm_peak: float) -> dict:
    """One workload's quantize step and GEMM, each timed on its own with CUDA
    events (L2 flushed before every timed launch, outside the events; the
    launches replayed from CUDA graphs); medians over `reps`."""
    idx, shape_index = WORKLOADS[name]
    wl = W.make_workload(idx, shape_index)
    st = make_step(wl, dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    for _ in range(3):
        st.quantize()
        st.gemm()
    torch.cuda.synchronize()
    st.f.check_device_status()
    gq = capture(st.quantize)
    gg = capture(st.gemm, pool=gq.pool())
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(reps)]
    for i in range(reps):
        evict_l2(flush)
        ev[i][0].record(stream)
        gq.replay()
        ev[i][1].record(stream)
        evict_l2(flush)
        ev[i][2].record(stream)
        gg.replay()
        ev[i][3].record(stream)
    torch.cuda.synchronize()
    st.f.check_device_status()
    q_us = float(np.median([e[0].elapsed_time(e[1]) for e in ev])) * 1e3
    g_us = float(np.median([e[2].elapsed_time(e[3]) for e in ev])) * 1e3
    qbytes = st.quant_bytes()
    out = {"M": wl.M, "N": wl.N, "K": wl.K, "recipe": wl.recipe, "E": wl.E or None,
           "gemm_us": g_us, "quantize_us": q_us, "reps": reps}
    if name == "tensorwise_256":
        out["note"] = "launch-latency bound (33.6 MFLOP): microseconds only"
    else:
        tf = wl.flops / (g_us * 1e-6) / 1e12
        gbs = qbytes / (q_us * 1e-6) / 1e9
        out.update({"gemm_tflops": tf, "gemm_frac": tf / fp8_peak,
                    "gemm_frac_nominal": tf / NOMINAL_FP8_TFLOPS,
                    "quantize_gbs": gbs, "quantize_frac": gbs / hbm_peak,
                    "quantize_bytes": qbytes})
    del gq, gg, st, flush
    torch.cuda.empty_cache()
    return out


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


DENSE_RECIPES = ("tensor", "row", "1x128_128x128", "1x128_128x1")
_B_CODES = {}   # oracle codes of a workload's B operand, made once per process


def oracle_dense_sample(wl, rows: int):
    """A proportional slice of one step of a dense workload on the CPU
    oracle: quantize rows [0, r) of A and the matching share of B's rows
    (rounded up to whole 128-row groups), then the GEMM of output rows
    [0, r) (against B's codes for all N rows, made once, untimed).  Returns
    (quantize seconds, GEMM seconds, the step's fraction r/M, threads)."""
    import oracle
    ga, gb = OPERAND_GROUPS[wl.recipe]
    G = {"tensor": oracle.GROUP_TENSOR, "row": oracle.GROUP_ROW,
         "1x128": oracle.GROUP_1x128, "128x128": oracle.GROUP_128x128}
    MMR = {"tensor": oracle.MM_TENSOR_TENSOR, "row": oracle.MM_ROW_ROW,
           "1x128_128x128": oracle.MM_1x128_128x128, "1x128_128x1": oracle.MM_1x128_128x1}
    r = int(max(1, min(wl.M, rows)))
    key = (id(wl), wl.recipe)
    if key not in _B_CODES:
        _B_CODES.clear()
        _B_CODES[key] = oracle.quantize(W.bf16_bits(wl.b), G[gb])
    qb, sb = _B_CODES[key]
    rb = min(wl.N, -(-(r * wl.N // wl.M + 1) // 128) * 128)
    abits, bbits = W.bf16_bits(wl.a[:r]), W.bf16_bits(wl.b[:rb])
    t0 = time.perf_counter()
    qa, sa = oracle.quantize(abits, G[ga])
    oracle.quantize(bbits, G[gb])
    tq = time.perf_counter() - t0
    bias = None if wl.bias is None else W.bf16_bits(wl.bias)
    t0 = time.perf_counter()
    oracle.scaled_mm(qa, qb, sa, sb, MMR[wl.recipe], bias_bits=bias)
    tg = time.perf_counter() - t0
    return tq, tg, r / wl.M, oracle.num_threads()


def sample_rows(wl, flop_budget: float = 6e10) -> int:
    """Output rows of the oracle's sample: about `flop_budget` of GEMM work
    (a second or two on a 16-core host), at least 8 rows (a whole 128-token
    group for the training step), at most all of them.  Fixed by the
    workload alone, so both benchmark arms time the same sample."""
    per_row = wl.flops / max(1, wl.M)
    r = int(round(flop_budget / per_row))
    if wl.recipe == "chain_train":
        return int(min(wl.M, max(128, -(-r // 128) * 128)))
    return int(max(8, min(wl.M, r)))


def cpu_baseline(wl, rows: int, repeats: int = 1):
    """The oracle timed on a bounded sample of one step of the workload.
    Dense recipes: a proportional slice of the step (quantize and GEMM of
    r/M of it), value = the slice's GEMM FLOPs / its time.  Other recipes:
    quantize of the operands in full plus the GEMM on the first rows, the
    GEMM time scaled to all rows."""
    if wl.recipe in DENSE_RECIPES:
        vals, secs = [], []
        for _ in range(repeats):
            tq, tg, frac, threads = oracle_dense_sample(wl, rows)
            secs.append(tq + tg)
            vals.append(frac * wl.flops / (tq + tg) / 1e12)
        r = int(round(frac * wl.M))
        return {"value": float(np.median(vals)), "unit": "TFLOP/s", "cores": threads,
                "kind": "oracle", "extrapolated": True, "sample_rows": r,
                "sample": (f"rows 0..{r} of {wl.M}: quantize of those rows of A and of the "
                           f"matching share of B's rows, then the GEMM of those output rows "
                           f"({float(np.median(secs)):.2f} s, {r / wl.M:.4f} of the step); "
                           f"the rate over the slice, scaled to all rows"),
                "seconds_per_sample": float(np.median(secs)),
                "seconds_est_per_step": float(np.median(secs)) * wl.M / r}
    tg, frac, tq, threads = oracle_sample(wl, rows)
    est_s = tq + tg / frac
    value = wl.flops / est_s / 1e12
    r = int(round(frac * wl.M))
    common = {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
              "extrapolated": True, "sample_rows": r, "seconds_per_sample": tq + tg,
              "seconds_est_per_step": est_s}
    if wl.recipe == "chain_train":
        return dict(common, sample=(
            f"quantize of W1 and W2, as stored and transposed, in full "
            f"({tq:.2f} s) + the rest of the step (activation quantizes, six "
            f"GEMMs, both quantized forms of Y1 and dY1) on the first {r} of "
            f"{wl.M} tokens ({tg:.2f} s), scaled to all rows"))
    chain = wl.recipe in ("chain", "chain_mx")
    what = "X, W1 and W2" if chain else "both operands"
    gemm = (("both GEMMs (the first one's fp32 output quantized "
             + ("MXFP8)" if wl.recipe == "chain_mx" else "1x128)")) if chain else "GEMM")
    return dict(common, sample=(
        f"quantize of {what} in full ({tq:.2f} s) + {gemm} on {r} of {wl.M} output "
        f"rows ({tg:.2f} s), scaled to all rows"))


# ------------------------------------------------------------ kernel tables

def _timed_graph(fn, reps: int, flush: torch.Tensor) -> float:
    """Median device time (µs) of `fn`'s launches replayed from a CUDA graph,
    L2 flushed before every replay (outside the events)."""
    from fp8_scaled_matrix_b200 import fp8sm
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        evict_l2(flush)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) * 1e3)
    fp8sm.check_device_status()
    return float(np.median(ts))


def _random_codes(r: int, c: int, dev) -> torch.Tensor:
    """e4m3 codes of random finite values (no NaN codes)."""
    x = torch.randint(0, 0x7E, (r, c), dtype=torch.int32, device=dev)
    s = torch.randint(0, 2, (r, c), dtype=torch.int32, device=dev) << 7
    return (x | s).to(torch.uint8)


def kernel_table(kind: str, only, dev, reps: int = 30) -> dict:
    """Every quantize kernel (kind "quantize") or GEMM recipe (kind "gemm")
    timed alone on the benchmark's shapes: one launch per CUDA-graph replay,
    L2 flushed before each, median of `reps`.  Quantize inputs are N(0,1) bf16
    (codes and scales do not change the time); GEMM inputs are random e4m3
    codes with random positive scales."""
    from fp8_scaled_matrix_b200 import fp8sm
    torch.manual_seed(0)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    peaks, _ = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    fp8_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])) * FP8_OVER_BF16
    res = {}

    def want(name):
        return not only or name in only

    if kind == "quantize":
        R = {"tensor": fp8sm.FP8_SCALE_TENSOR, "row": fp8sm.FP8_SCALE_ROW,
             "1x128": fp8sm.FP8_SCALE_BLOCK_1x128, "128x128": fp8sm.FP8_SCALE_BLOCK_128x128}

        def rec(name, nbytes, fn):
            us = _timed_graph(fn, reps, flush)
            res[name] = {"us": us, "gbs": nbytes / us / 1e3, "frac": nbytes / us / 1e3 / hbm}

        def bf16(r, c):
            return torch.randn(r, c, device=dev).to(torch.bfloat16)
        for rows, cols, rc in [(4096, 4096, "row"), (32768, 4096, "row"), (65536, 4096, "row"),
                               (16640, 8192, "1x128"), (16640, 5120, "1x128"),
                               (5120, 8192, "128x128"), (8192, 5120, "128x128"),
                               (256, 256, "tensor")]:
            name = f"{rc}_{rows}x{cols}"
            if not want(name):
                continue
            t = bf16(rows, cols)
            q = torch.empty(rows, cols, dtype=torch.uint8, device=dev)
            sc = torch.empty(max(fp8sm.scale_count(rows, cols, R[rc]), 1), dtype=torch.float32,
                             device=dev)
            ws = torch.zeros(64, dtype=torch.uint8, device=dev)
            rec(name, 3 * rows * cols + 4 * sc.numel(),
                lambda: fp8sm.fp8_quantize(t, R[rc], out=q, scales=sc, workspace=ws))
        for rows, cols, rc in [(16640, 8192, "1x128"), (16640, 5120, "1x128"),
                               (5120, 8192, "128x128"), (8192, 5120, "128x128")]:
            name = f"T{rc}_{rows}x{cols}"
            if not want(name):
                continue
            t = bf16(rows, cols)
            q = torch.empty(cols, rows, dtype=torch.uint8, device=dev)
            n = ((rows // 128) * cols if rc == "1x128"
                 else (rows // 128) * ((cols + 127) // 128))
            sc = torch.empty(n, dtype=torch.float32, device=dev)
            rec(name, 3 * rows * cols + 4 * n,
                lambda: fp8sm.fp8_quantize_transposed(t, R[rc], out=q, scales=sc))
        if want("Tgrouped_32768x4096"):
            wl = W.make_workload(13, 0)   # the MoE weight gradient's tokens and split
            t, offs = wl.a.to(dev), wl.offs.to(dev)
            P = fp8sm.fp8_grouped_padded_tokens(wl.K, wl.E)
            q = torch.empty(wl.M, P, dtype=torch.uint8, device=dev)
            sc = torch.empty(P // 128, wl.M, dtype=torch.float32, device=dev)
            rec("Tgrouped_32768x4096", 3 * t.numel() + 4 * sc.numel(),
                lambda: fp8sm.fp8_quantize_transposed_grouped(t, offs, out=q, scales=sc))
        if want("batched128_16x4096x4096") or want("Tbatched128_16x4096x4096"):
            t = (torch.randn(16 * 4096, 4096, device=dev) * 0.02).to(torch.bfloat16)
            t = t.view(16, 4096, 4096)
            q = torch.empty(16 * 4096, 4096, dtype=torch.uint8, device=dev)
            sc = torch.empty(16 * 32 * 32, dtype=torch.float32, device=dev)
            nb = 3 * t.numel() + 4 * sc.numel()
            if want("batched128_16x4096x4096"):
                rec("batched128_16x4096x4096", nb, lambda: fp8sm.fp8_quantize_batched(
                    t, fp8sm.FP8_SCALE_BLOCK_128x128, out=q, scales=sc))
            if want("Tbatched128_16x4096x4096"):
                rec("Tbatched128_16x4096x4096", nb, lambda: fp8sm.fp8_quantize_transposed_batched(
                    t, fp8sm.FP8_SCALE_BLOCK_128x128, out=q, scales=sc))
        if want("mx_16640x8192"):
            t = bf16(16640, 8192)
            q = torch.empty(16640, 8192, dtype=torch.uint8, device=dev)
            sc = torch.empty(fp8sm.fp8_mx_scale_bytes(16640, 8192), dtype=torch.uint8, device=dev)
            rec("mx_16640x8192", 3 * t.numel() + sc.numel(),
                lambda: fp8sm.fp8_quantize_mx(t, out=q, scales=sc))
        return res

    def gemm(name, M, N, K, recipe):
        if not want(name):
            return
        a, b = _random_codes(M, K, dev), _random_codes(N, K, dev)
        if recipe == "1x128_128x128":
            na, nb = (K // 128) * M, (K // 128) * ((N + 127) // 128)
        elif recipe == "1x128_128x1":
            na, nb = (K // 128) * M, (K // 128) * N
        else:
            na, nb = M, N
        sa = torch.rand(na, device=dev) * 0.01 + 0.001
        sb = torch.rand(nb, device=dev) * 0.01 + 0.001
        out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        us = _timed_graph(lambda: fp8sm.fp8_scaled_mm(a, b, sa, sb, fp8sm.MM_RECIPES[recipe],
                                                      out=out), reps, flush)
        tf = 2 * M * N * K / us / 1e6
        res[name] = {"us": us, "tflops": tf, "frac": tf / fp8_peak}
    gemm("blk128", 16640, 5120, 8192, "1x128_128x128")
    gemm("blk128_b", 16640, 8192, 5120, "1x128_128x128")
    gemm("blk1", 16640, 5120, 8192, "1x128_128x1")
    gemm("blk1_b", 16640, 8192, 5120, "1x128_128x1")
    gemm("row", 4096, 4096, 4096, "row")
    gemm("row_16640x5120x8192", 16640, 5120, 8192, "row")
    if want("mx"):
        M, N, K = 16640, 5120, 8192
        a, b = _random_codes(M, K, dev), _random_codes(N, K, dev)
        sa = torch.randint(120, 130, (fp8sm.fp8_mx_scale_bytes(M, K),), dtype=torch.uint8,
                           device=dev)
        sb = torch.randint(120, 130, (fp8sm.fp8_mx_scale_bytes(N, K),), dtype=torch.uint8,
                           device=dev)
        out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        us = _timed_graph(lambda: fp8sm.fp8_scaled_mm_mx(a, b, sa, sb, out=out), reps, flush)
        tf = 2 * M * N * K / us / 1e6
        res["mx"] = {"us": us, "tflops": tf, "frac": tf / fp8_peak}
    return res


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
                    help="output rows of the CPU oracle's sample (0: a fixed share of the "
                         "workload, the same in both arms)")
    ap.add_argument("--no-all-configs", action="store_true",
                    help="skip timing the five benchmark configurations after the step")
    ap.add_argument("--config-reps", type=int, default=20)
    ap.add_argument("--kernel-table", choices=["quantize", "gemm"], default=None,
                    help="time every quantize kernel or GEMM recipe alone on the benchmark's "
                         "shapes and print one JSON line with the table (no step)")
    ap.add_argument("--only", default="",
                    help="with --kernel-table: comma-separated entry names to time")
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
        steps = args.steps or 3
        rows = args.cpu_rows or sample_rows(wl)
        # every step is the same bounded sample of the workload's step (the
        # oracle run as it stands); warm-up samples are not timed
        for _ in range(args.warmup):
            cpu_baseline(wl, rows)
        samples = []
        t_run = time.perf_counter()
        for _ in range(steps):
            samples.append(cpu_baseline(wl, rows))
        t_run = time.perf_counter() - t_run
        value = float(np.mean([b["value"] for b in samples]))
        b = samples[-1]
        line = {
            "impl": "reference", "metric": "fp8_scaled_gemm_tflops", "value": value,
            "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup,
            "ms_per_step": t_run / steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp8e4m3/int64-exact/f64", "data": "synthetic",
            "config": {"workload": args.workload, "M": wl.M, "N": wl.N, "K": wl.K},
            "extrapolated": True,
            "sample_rows": b["sample_rows"],
            "est_full_step_ms": float(np.mean([x["seconds_est_per_step"] for x in samples])) * 1e3,
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": b["cores"],
                             "kind": "oracle", "sample": b["sample"],
                             "sample_rows": b["sample_rows"], "extrapolated": True},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return 0

    if args.kernel_table:
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        from fp8_scaled_matrix_b200 import build
        build.build()
        only = [x for x in args.only.split(",") if x]
        print(json.dumps({"kernel_table": args.kernel_table,
                          "entries": kernel_table(args.kernel_table, only, dev)}), flush=True)
        return 0

    if world > 1:
        torch.cuda.set_device(local_rank)
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local_rank)
    from fp8_scaled_matrix_b200 import build
    build.build()

    wl = W.make_workload(idx, shape_index)
    if world > 1:
        wl.a = rank_shard_rows(wl.a, rank, world)
    if args.steps is None:
        # about a second of timed work per workload
        args.steps = {"tensorwise_256": 4000, "rowwise_4096": 3000,
                      "grouped_e16": 1000}.get(args.workload, 600)
    peaks, peak_src = load_peaks()
    fp8_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])) * FP8_OVER_BF16
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    sampler = ClockSampler(dev)
    sampler.start()
    try:
        res = run_ours(args, wl, dev, rank, world, sampler)
        configs = None
        if world == 1 and not args.no_all_configs:
            t0 = time.perf_counter()
            configs = {name: measure_config(name, dev, args.config_reps, fp8_peak, hbm_peak)
                       for name in ALL_CONFIGS}
            configs["clocks"] = sampler.window(t0, time.perf_counter())
    finally:
        sampler.stop()

    K = args.steps
    ms_per_step = res["total_ms"] / K
    value = job_tflops(wl.flops, world, ms_per_step)
    gemm_tflops = wl.flops / (res["g_ms"] * 1e-3) / 1e12
    quant_gbs = res["quant_bytes"] / (res["q_ms"] * 1e-3) / 1e9
    traffic = recorded_traffic(args.workload)
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
            "step": ("quantize W1, W2, then X (one stream), then GEMM1 with its "
                     "output quantized 1x128 in the epilogue, then GEMM2"
                     if wl.recipe == "chain" else
                     "MXFP8 quantize X || W1, W2 (two streams), then GEMM1 with MXFP8 "
                     "output, then GEMM2" if wl.recipe == "chain_mx" else
                     "quantize X, X^T, dY2, dY2^T || W1, W2, W1^T, W2^T (two streams), then "
                     "the chain's forward (Y1 = X W1^T writing Y1 and Y1^T in e4m3, Y2 = Y1 "
                     "W2^T) and backward (dY1 = dY2 W2 writing dY1 and dY1^T in e4m3, dX = "
                     "dY1 W1, dW1 = dY1^T X, dW2 = dY2^T Y1)"
                     if wl.recipe == "chain_train" else
                     "quantize B, then A (one stream), then scaled GEMM"
                     if wl.recipe == "1x128_128x128" else
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
            "traffic": traffic,
            "traffic_source": ("ncu capture of this GEMM kernel's sources "
                               "(profiles/dram_traffic.json), not measured in this run"
                               if traffic is not None else
                               "none recorded for the current GEMM kernel sources"),
            "kernel": "fp8_gemm_kernel", "peak_source":
                f"{peak_src} bf16 burst x {FP8_OVER_BF16:g} (nominal fp8/bf16 dense ratio)",
            "peak_nominal": NOMINAL_FP8_TFLOPS,
            "frac_nominal": gemm_tflops / NOMINAL_FP8_TFLOPS,
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
    if configs is not None:
        line["all_configs"] = configs
    if "e2e" in res:
        e = res["e2e"]
        line["e2e"] = {"value": job_tflops(wl.flops, world, e["ms"]), "unit": "TFLOP/s",
                       "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"],
                       "ms_per_step": e["ms"], "steps": e["steps"]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = args.cpu_rows or sample_rows(wl)
        cb = cpu_baseline(wl, rows, repeats=2)
        line["cpu_baseline"] = {k: v for k, v in cb.items()
                                if k not in ("seconds_est_per_step", "seconds_per_sample")}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
