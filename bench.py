#!/usr/bin/env python
"""Benchmark of the binarized linear layers on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|prefill|backward|w1a8|w1a8_single|w158a8|w1a8_tensor|w1a1|
                                decode_stack|decode_stack16]
                    [--no-secondary] [--probe-int8]

Workloads (a step is one pass of the layer over one batch of synthetic input):

* ``decode`` (default, the headline): FBI-linear W1A16 GEMV, M=1 token,
  K=N=4096 (a 7B attention projection), judged on packed-weight bytes per
  second against the measured HBM bandwidth;
* ``prefill``: FBI-linear W1A16 on the 7B MLP shapes, 2048 tokens, the
  up-projection 4096->11008 then the down-projection 11008->4096, judged in
  TFLOP/s against the measured bf16 tensor peak;
* ``w1a8``: BitNet BitLinear (LN + absmax int8 quantisation + int8 GEMM +
  rescale) on the 1.3B shapes, 512 tokens, 2048->5632 then 5632->2048, in
  TOP/s against the int8 tensor peak;
* ``w158a8``: the same with BitNet b1.58 ternary weights;
* ``w1a8_tensor``: the same with the per-tensor Eq.(5) quantiser;
* ``w1a1``: XNOR/popcount products of packed +-1 operands at the same shapes,
  against a population-count (integer ALU) roofline;
* ``w1a8_single``: one small BitLinear layer, M=4 tokens, K=N=256 (one fused
  launch), in tokens per second;
* ``backward``: the straight-through FBI-linear backward (dx, dW, dalpha) of
  the 7B MLP up-projection at 2048 tokens, in TFLOP/s;
* ``decode_stack`` / ``decode_stack16``: one token step of a 7B-shaped
  FBI-LLM's 224 linears (32 layers, each layer's outputs feeding the next) at
  batch 1 / 16 as one stacked call, in tokens per second, against HBM.

Each workload keeps R distinct copies of its weights and activations whose
total is more than twice the 126 MB L2, and step i uses copy i % R, so no step
finds its inputs in L2 (the stacked decode streams 0.8 GB of signs per step:
one copy). After W untimed warm-up steps, K steps are captured
in one CUDA graph and timed with CUDA events recorded as the graph's first and
last nodes on the launching stream; with N
ranks (torchrun) every rank runs its own replica (no data-path collective)
and the time is the max over ranks.

Rank 0 prints one JSON line. `--impl reference` times the CPU oracle on a
bounded sample of the same workload instead (the reference arm).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CSRC = "bit_linear_layers_b200/csrc/"
SUSTAINED_AFTER_S = 1.0  # a timed region longer than this runs under the power cap: sustained peak


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode", choices=sorted(WORKLOADS))
    ap.add_argument("--probe-int8", action="store_true",
                    help="measure the dense int8 tensor throughput of this GPU (torch._int_mm, 8192^3) and exit")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the other workloads and the 7B measurement that ride along at N=1")
    a = ap.parse_args()
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    return a


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def src_hash(sources) -> str:
    h = hashlib.sha256()
    for rel in sources:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


class ClockSampler:
    """nvidia-smi clock/throttle samples every 100 ms while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.out = tempfile.TemporaryFile(mode="w+")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.seek(0)
        rows = [r.split(",") for r in self.out.read().strip().splitlines() if r.strip()]
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 8:
                continue
            try:
                sm.append(float(r[0]))
                mx = max(mx, float(r[1]))
            except ValueError:
                continue
            for name, v in zip(names, r[4:8]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "window": "warm-up and timed steps"}


# ----------------------------------------------------------------------------- workloads


class Workload:
    """One benchmarked configuration: its rotating device copies, a device
    step, an end-to-end step through pinned host buffers, and the oracle's
    bounded sample of the same work."""

    name = ""
    metric = ""
    unit = ""
    scale = 1e9          # unit = work units per second / scale
    dtype = "bf16"
    bound = "hbm"
    kernel = ""
    sources: list = []
    traffic_file = None
    launches_per_step = 1
    rotate = 1
    config: dict = {}

    def units_per_step(self) -> float:
        raise NotImplementedError

    def achieved(self, per_step_s: float) -> float:
        """Algorithmic bytes (or flops) of the dominant kernel per launch over its launch time."""
        return self.units_per_step() / per_step_s / self.scale

    def peak(self, peaks, timed_s):
        raise NotImplementedError

    def traffic(self):
        """DRAM bytes per launch from the committed ncu summary, or None when
        the summary is missing or was taken on another version of the kernel."""
        if self.traffic_file is None:
            return None
        path = os.path.join(ROOT, "profiles", self.traffic_file)
        if not os.path.exists(path):
            return None
        with open(path) as f:
            d = json.load(f)
        if d.get("src_hash") != src_hash(self.sources):
            return None
        return d.get("dram_bytes_per_launch", d.get("dram_bytes_per_step"))


class Decode(Workload):
    name = "decode"
    M, K, N = 1, 4096, 4096
    metric = "decode GEMV HBM GB/s on packed-weight bytes (W1A16, 1x4096x4096)"
    unit, scale, bound = "GB/s", 1e9, "hbm"
    kernel = "gemv_w1a16_lut_kernel<1> (cluster of 8 x 16 clusters)"
    sources = [CSRC + "bl_gemv_lut.cuh", CSRC + "bl_common.cuh", CSRC + "bl_api.cu"]
    traffic_file = "gemv_w1a16_decode_1x4096x4096.traffic.json"
    rotate = 128

    def __init__(self):
        self.packed_b = self.N * self.K // 8
        self.alg_b = self.packed_b + 4 * self.N + 2 * self.M * self.K + 2 * self.M * self.N
        self.config = {"workload": "FBI-linear W1A16 decode GEMV, M=1, K=4096, N=4096 (7B attention projection)",
                       "M": self.M, "K": self.K, "N": self.N,
                       "l2": f"inputs larger than L2: {self.rotate} distinct packed weight copies "
                             f"({self.rotate * self.packed_b / 1e6:.0f} MB) rotated step to step",
                       "launch": "programmatic dependent launch between steps (BL_FLAG_OVERLAP_PREVIOUS)"}

    def units_per_step(self):
        return self.packed_b  # the metric counts packed-weight bytes

    def achieved(self, per_step_s):
        return self.alg_b / per_step_s / 1e9  # all bytes the kernel must move

    def peak(self, peaks, timed_s):
        return peaks["hbm_gbs"], "hbm_gbs"

    def setup(self, dev, rank):
        import torch
        import bit_linear_layers_b200 as bl
        import synthetic
        self.bl = bl
        self.packs, self.alphas, self.xs = [], [], []
        for i in range(self.rotate):
            if i == 0:  # the seeded workload itself (CPU generator)
                W = synthetic.weights(self.N, self.K, seed=2).to(dev)
                x = synthetic.activations(self.M, self.K, seed=2).to(dev)
            else:       # further seeded draws made on the device
                W = synthetic.weights(self.N, self.K, seed=replica_seed(2, i, rank), device=dev)
                x = synthetic.activations(self.M, self.K, seed=replica_seed(2, i, rank), device=dev)
            p, a = bl.bin_pack(W, bl.BL_PACK_FBI)
            self.packs.append(p)
            self.alphas.append(a)
            self.xs.append(x)
            del W
        self.ys = [torch.empty((self.M, self.N), dtype=torch.bfloat16, device=dev) for _ in range(self.rotate)]
        # consecutive steps never write each other's inputs, so each launch may
        # start streaming its weights while the previous one finishes
        self.flags = bl.BL_FLAG_OVERLAP_PREVIOUS
        self.xh = [x.cpu().pin_memory() for x in self.xs]
        self.yh = [torch.empty((self.M, self.N), dtype=torch.bfloat16).pin_memory() for _ in range(self.rotate)]
        self.xd = torch.empty((self.M, self.K), dtype=torch.bfloat16, device=dev)
        self.yd = torch.empty((self.M, self.N), dtype=torch.bfloat16, device=dev)
        self.h2d, self.d2h = 2 * self.M * self.K, 2 * self.M * self.N

    def step(self, i):
        j = i % self.rotate
        self.bl.bin_linear_w1a16(self.xs[j], self.packs[j], self.alphas[j], out=self.ys[j], flags=self.flags)

    def e2e_step(self, i):
        j = i % self.rotate
        self.xd.copy_(self.xh[j], non_blocking=True)
        self.bl.bin_linear_w1a16(self.xd, self.packs[j], self.alphas[j], out=self.yd, flags=self.flags)
        self.yh[j].copy_(self.yd, non_blocking=True)

    # oracle: output rows [0, 1024) of the decode problem per call
    ORACLE_ROWS = 1024

    def oracle_setup(self):
        import oracle as oracle_pkg
        import synthetic
        self.o = oracle_pkg.get()
        W = synthetic.weights(self.N, self.K, seed=2).numpy()
        self.ox = synthetic.bf16_bits(synthetic.activations(self.M, self.K, seed=2))
        packed, alpha = self.o.pack_fbi(W)
        self.op, self.oa = packed[:self.ORACLE_ROWS].copy(), alpha[:self.ORACLE_ROWS].copy()
        self.oracle_sample = (f"output rows 0..{self.ORACLE_ROWS - 1} of the 1x4096x4096 problem per call "
                              "(single-threaded C oracle, fp64)")
        return self.ORACLE_ROWS * self.K / 8  # units (packed bytes) per call

    def oracle_call(self):
        self.o.w1a16(self.ox, self.op, self.oa, self.K)


class Prefill(Workload):
    name = "prefill"
    SHAPES = [(2048, 4096, 11008), (2048, 11008, 4096)]  # (M, K, N)
    metric = "prefill TFLOP/s (W1A16, 7B MLP up + down projections, 2048 tokens)"
    unit, scale, bound = "TFLOP/s", 1e12, "tensor"
    kernel = "gemm_ts_kernel<0,1,256,false> (persistent, 148 CTAs)"
    sources = [CSRC + "bl_gemm_ts.cuh", CSRC + "bl_common.cuh", CSRC + "bl_api.cu"]
    traffic_file = "gemm_ts_w1a16_prefill_2048x4096x11008.traffic.json"
    launches_per_step = 2
    rotate = 4

    def __init__(self):
        per_copy = sum(M * K * 2 + N * K // 8 + 4 * N + M * N * 2 for M, K, N in self.SHAPES)
        self.config = {"workload": "FBI-linear W1A16 prefill GEMM, 2048 tokens, 7B MLP shapes "
                                   "4096->11008 then 11008->4096",
                       "shapes_MKN": [list(s) for s in self.SHAPES],
                       "l2": f"inputs larger than L2: {self.rotate} distinct copies of weights, activations "
                             f"and outputs ({self.rotate * per_copy / 1e6:.0f} MB) rotated step to step"}

    def units_per_step(self):
        return sum(2.0 * M * K * N for M, K, N in self.SHAPES)

    def peak(self, peaks, timed_s):
        key = "bf16_tflops_sustained" if timed_s > SUSTAINED_AFTER_S else "bf16_tflops"
        return peaks[key], key

    def setup(self, dev, rank):
        import torch
        import bit_linear_layers_b200 as bl
        import synthetic
        self.bl = bl
        self.copies = []
        for i in range(self.rotate):
            layers = []
            for s, (M, K, N) in enumerate(self.SHAPES):
                seed = 1 + 100 * i + 10 * s + 7 * rank
                W = synthetic.weights(N, K, seed=seed, device=dev)
                p, a = bl.bin_pack(W, bl.BL_PACK_FBI)
                del W
                x = synthetic.activations(M, K, seed=seed, device=dev)
                y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
                layers.append((x, p, a, y))
            self.copies.append(layers)
        self.xh = [lay[0].cpu().pin_memory() for lay in self.copies[0]]
        self.yh = [torch.empty_like(lay[3], device="cpu").pin_memory() for lay in self.copies[0]]
        self.h2d = sum(M * K * 2 for M, K, N in self.SHAPES)
        self.d2h = sum(M * N * 2 for M, K, N in self.SHAPES)

    def step(self, i):
        for x, p, a, y in self.copies[i % self.rotate]:
            self.bl.bin_linear_w1a16(x, p, a, out=y)

    def e2e_step(self, i):
        for (x, p, a, y), xh, yh in zip(self.copies[i % self.rotate], self.xh, self.yh):
            x.copy_(xh, non_blocking=True)
            self.bl.bin_linear_w1a16(x, p, a, out=y)
            yh.copy_(y, non_blocking=True)

    # oracle: one token through output columns [0, 512) of the up and [0, 256) of the down projection
    ORACLE_COLS = (512, 256)

    def oracle_setup(self):
        import oracle as oracle_pkg
        import synthetic
        self.o = oracle_pkg.get()
        self.olayers, flop = [], 0.0
        for s, ((M, K, N), cols) in enumerate(zip(self.SHAPES, self.ORACLE_COLS)):
            W = synthetic.weights(cols, K, seed=1 + 10 * s).numpy()  # `cols` rows of a seeded layer
            x = synthetic.bf16_bits(synthetic.activations(1, K, seed=1 + 10 * s))
            p, a = self.o.pack_fbi(W)
            self.olayers.append((x, p, a, K))
            flop += 2.0 * K * cols
        self.oracle_sample = ("one token through output columns 0..511 of the up and 0..255 of the down "
                              "projection per call (single-threaded C oracle, fp64)")
        return flop

    def oracle_call(self):
        for x, p, a, K in self.olayers:
            self.o.w1a16(x, p, a, K)


class Backward(Workload):
    """Straight-through backward of FBI-linear at the 7B MLP up-projection
    shape (2048 tokens, 4096 -> 11008): dx, dW and dalpha per step."""
    name = "backward"
    M, K, N = 2048, 4096, 11008
    metric = "FBI-linear STE backward TFLOP/s (dx + dW, 7B MLP up-projection, 2048 tokens)"
    unit, scale, bound = "TFLOP/s", 1e12, "tensor"
    kernel = ("gemm_ts_kernel<0,1,256,false> (dx on transposed signs) + gemm_ss_ste_kernel (dW) + "
              "layout kernels (one call)")
    sources = [CSRC + "bl_backward.cuh", CSRC + "bl_gemm_ts.cuh", CSRC + "bl_common.cuh", CSRC + "bl_api.cu"]
    traffic_file = "ste_backward_2048x4096x11008.traffic.json"  # the dx GEMM launch (largest share of the step)
    launches_per_step = 8  # split, transposed pack, fill, dx GEMM, two transposes, dW GEMM, finalize
    rotate = 2

    def __init__(self):
        M, K, N = self.M, self.K, self.N
        per_copy = M * K * 2 + M * N * 2 + N * K // 8 + 4 * N + M * K * 2 + N * K * 4 + 4 * N
        self.config = {"workload": "FBI-linear straight-through backward, 2048 tokens, 7B MLP up-projection "
                                   "4096->11008 (dx bf16, dW fp32, dalpha fp32)",
                       "M": M, "K": K, "N": N,
                       "l2": f"inputs larger than L2: {self.rotate} distinct copies of x, dy, weights, gradients "
                             f"and workspaces ({self.rotate * per_copy / 1e6:.0f} MB plus workspaces) rotated"}

    def units_per_step(self):
        return 2.0 * (2.0 * self.M * self.N * self.K)  # the dx and dW contractions

    def peak(self, peaks, timed_s):
        key = "bf16_tflops_sustained" if timed_s > SUSTAINED_AFTER_S else "bf16_tflops"
        return peaks[key], key

    def setup(self, dev, rank):
        import torch
        import bit_linear_layers_b200 as bl
        import synthetic
        self.bl = bl
        M, K, N = self.M, self.K, self.N
        self.copies = []
        for i in range(self.rotate):
            seed = 3 + 100 * i + 7 * rank
            W = synthetic.weights(N, K, seed=seed, device=dev)
            p, a = bl.bin_pack(W, bl.BL_PACK_FBI)
            del W
            x = synthetic.activations(M, K, seed=seed, device=dev)
            dy = synthetic.activations(M, N, seed=seed + 1, device=dev)
            dx = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
            dw = torch.empty((N, K), dtype=torch.float32, device=dev)
            da = torch.empty(N, dtype=torch.float32, device=dev)
            ws = torch.empty(bl.workspace_bytes(bl.BL_OP_W1A16_BACKWARD, M, N, K), dtype=torch.uint8, device=dev)
            self.copies.append((x, dy, p, a, dx, dw, da, ws))
        c = self.copies[0]
        self.xh, self.dyh = c[0].cpu().pin_memory(), c[1].cpu().pin_memory()
        self.dxh = torch.empty_like(c[4], device="cpu").pin_memory()
        self.dwh = torch.empty_like(c[5], device="cpu").pin_memory()
        self.dah = torch.empty_like(c[6], device="cpu").pin_memory()
        self.h2d = M * K * 2 + M * N * 2
        self.d2h = M * K * 2 + N * K * 4 + N * 4

    def step(self, i):
        x, dy, p, a, dx, dw, da, ws = self.copies[i % self.rotate]
        self.bl.bin_linear_w1a16_backward(x, p, a, dy, dx=dx, dw=dw, dalpha=da, ws=ws)

    def e2e_step(self, i):
        x, dy, p, a, dx, dw, da, ws = self.copies[i % self.rotate]
        x.copy_(self.xh, non_blocking=True)
        dy.copy_(self.dyh, non_blocking=True)
        self.bl.bin_linear_w1a16_backward(x, p, a, dy, dx=dx, dw=dw, dalpha=da, ws=ws)
        self.dxh.copy_(dx, non_blocking=True)
        self.dwh.copy_(dw, non_blocking=True)
        self.dah.copy_(da, non_blocking=True)

    # oracle: 64 entries of dx and 64 of dW at the full shape per call
    ORACLE_POINTS = 64

    def oracle_setup(self):
        import numpy as np
        import oracle as oracle_pkg
        import synthetic
        self.o = oracle_pkg.get()
        M, K, N = self.M, self.K, self.N
        W = synthetic.weights(N, K, seed=3).numpy()
        self.op, self.oa = self.o.pack_fbi(W)
        self.ox = synthetic.bf16_bits(synthetic.activations(M, K, seed=3))
        self.ody = synthetic.bf16_bits(synthetic.activations(M, N, seed=4))
        rng = np.random.default_rng(0)
        n = self.ORACLE_POINTS
        self.opts = (rng.integers(0, M, n), rng.integers(0, K, n), rng.integers(0, N, n), rng.integers(0, K, n))
        self.oracle_sample = (f"{n} entries of dx (each a sum over the 11008 outputs) and {n} of dW (each a sum "
                              "over the 2048 tokens) per call (single-threaded C oracle, fp64)")
        return 2.0 * n * N + 2.0 * n * M

    def oracle_call(self):
        ms, ks, js, ks2 = self.opts
        self.o.w1a16_backward_at(self.ox, self.op, self.oa, self.ody, self.K, "dx", ms, ks)
        self.o.w1a16_backward_at(self.ox, self.op, self.oa, self.ody, self.K, "dw", js, ks2)


class W1A8(Workload):
    name = "w1a8"
    SHAPES = [(512, 2048, 5632), (512, 5632, 2048)]
    metric = "BitLinear W1A8 TOP/s (1.3B shapes, 512 tokens, LN + absmax quant + int8 GEMM + rescale)"
    unit, scale, bound = "TOP/s", 1e12, "tensor"
    dtype = "s8"
    kernel = "ln_quant_kernel<NV> + gemm_ts_kernel<1,1,256|128,*> (one call; time includes LN + quantisation)"
    sources = [CSRC + "bl_gemm_ts.cuh", CSRC + "bl_lnquant.cuh", CSRC + "bl_common.cuh", CSRC + "bl_api.cu"]
    traffic_file = "bitlinear_w1a8_1p3b_512tokens.traffic.json"  # the GEMM launches' DRAM bytes
    launches_per_step = 4
    rotate = 16

    def __init__(self):
        per_copy = sum(M * K * 2 + N * K // 8 + M * K + 8 * M + M * N * 4 for M, K, N in self.SHAPES)
        self.config = {"workload": "BitNet BitLinear W1A8, 512 tokens, 1.3B shapes 2048->5632 then 5632->2048",
                       "shapes_MKN": [list(s) for s in self.SHAPES],
                       "l2": f"inputs larger than L2: {self.rotate} distinct copies of weights, activations, "
                             f"workspaces and outputs ({self.rotate * per_copy / 1e6:.0f} MB) rotated step to step"}

    def units_per_step(self):
        return sum(2.0 * M * K * N for M, K, N in self.SHAPES)

    def peak(self, peaks, timed_s):
        key = "bf16_tflops_sustained" if timed_s > SUSTAINED_AFTER_S else "bf16_tflops"
        return 2.0 * peaks[key], f"2 x {key} (nominal int8/bf16 ratio)"

    def setup(self, dev, rank):
        import torch
        import bit_linear_layers_b200 as bl
        import synthetic
        self.bl = bl
        self.copies = []
        for i in range(self.rotate):
            layers = []
            for s, (M, K, N) in enumerate(self.SHAPES):
                seed = 4 + 100 * i + 10 * s + 7 * rank
                W = synthetic.weights(N, K, seed=seed, mean=0.001, device=dev)
                p, _, b = bl.bin_pack(W, bl.BL_PACK_BITNET)
                del W
                x = synthetic.laplace_channel_activations(M, K, seed=seed, device=dev)
                ws = torch.empty(bl.workspace_bytes(self.ws_op(bl), M, N, K), dtype=torch.uint8, device=dev)
                y = torch.empty((M, N), dtype=torch.float32, device=dev)
                layers.append((x, p, b, ws, y))
            self.copies.append(layers)
        self.xh = [lay[0].cpu().pin_memory() for lay in self.copies[0]]
        self.yh = [torch.empty_like(lay[4], device="cpu").pin_memory() for lay in self.copies[0]]
        self.h2d = sum(M * K * 2 for M, K, N in self.SHAPES)
        self.d2h = sum(M * N * 4 for M, K, N in self.SHAPES)

    def ws_op(self, bl):
        return bl.BL_OP_W1A8

    def call(self, x, p, b, ws, y):
        self.bl.bitlinear_w1a8(x, p, b, out=y, ws=ws)

    def step(self, i):
        for x, p, b, ws, y in self.copies[i % self.rotate]:
            self.call(x, p, b, ws, y)

    def e2e_step(self, i):
        for (x, p, b, ws, y), xh, yh in zip(self.copies[i % self.rotate], self.xh, self.yh):
            x.copy_(xh, non_blocking=True)
            self.call(x, p, b, ws, y)
            yh.copy_(y, non_blocking=True)

    # oracle: token 0 through output columns [0, 1024) of both projections
    ORACLE_COLS = 1024

    def oracle_setup(self):
        import oracle as oracle_pkg
        import synthetic
        self.o = oracle_pkg.get()
        self.olayers, ops = [], 0.0
        for s, (M, K, N) in enumerate(self.SHAPES):
            W = synthetic.weights(N, K, seed=4 + 10 * s, mean=0.001).numpy()
            p, _, beta = self.o.pack_bitnet(W)  # beta needs the whole matrix
            x = synthetic.bf16_bits(synthetic.laplace_channel_activations(1, K, seed=4 + 10 * s))
            self.olayers.append((x, p[:self.ORACLE_COLS].copy(), beta, K))
            ops += 2.0 * K * self.ORACLE_COLS
        self.oracle_sample = ("one token through LN + quantisation and output columns 0..1023 of both "
                              "projections per call (single-threaded C oracle, fp64/int64)")
        return ops

    def oracle_call(self):
        for x, p, beta, K in self.olayers:
            self.o.w1a8(x, p, beta, K)


class W1A8Single(Workload):
    """BitNet BitLinear, one small layer: M=4 tokens, K=N=256, seed 0. The
    whole forward (LN, per-token absmax int8 quantisation, +-1 products,
    beta*gamma/128 rescale) is one fused launch; the problem is latency-bound
    (14 KB of operands), so the roofline fraction is tiny by construction."""
    name = "w1a8_single"
    M, K, N = 4, 256, 256
    metric = "BitLinear W1A8 single layer tokens/s (M=4, K=N=256, LN + absmax quant + int8 products + rescale)"
    unit, scale, bound = "tok/s", 1.0, "hbm"
    dtype = "s8"
    kernel = "bitlinear_small_kernel<4,false> (one fused launch per call)"
    sources = [CSRC + "bl_gemv.cuh", CSRC + "bl_lnquant.cuh", CSRC + "bl_common.cuh", CSRC + "bl_api.cu"]
    traffic_file = "bitlinear_small_w1a8_single_4x256x256.traffic.json"
    roof_unit = "GB/s"
    rotate = 18000  # 14 KB per copy: 250 MB, about twice the L2

    def __init__(self):
        M, K, N = self.M, self.K, self.N
        self.bytes_per_call = N * K // 8 + 2 * M * K + 4 * M * N + 4
        self.config = {"workload": "BitNet BitLinear W1A8 single layer, M=4 tokens, K=N=256, seed 0",
                       "M": M, "K": K, "N": N,
                       "l2": f"inputs larger than L2: {self.rotate} distinct copies of weights, activations and "
                             f"outputs ({self.rotate * self.bytes_per_call / 1e6:.0f} MB) rotated step to step",
                       "launch": "one fused kernel per call"}

    def units_per_step(self):
        return float(self.M)  # tokens

    def achieved(self, per_step_s):
        return self.bytes_per_call / per_step_s / 1e9  # bytes the call must move

    def peak(self, peaks, timed_s):
        return peaks["hbm_gbs"], "hbm_gbs"

    def setup(self, dev, rank):
        import torch
        import bit_linear_layers_b200 as bl
        import synthetic
        self.bl = bl
        M, K, N = self.M, self.K, self.N
        # copy 0 is the seeded workload; the others are further seeded draws made on the device
        W = synthetic.weights(N * self.rotate, K, seed=replica_seed(0, 1, rank), device=dev)
        W[:N] = synthetic.weights(N, K, seed=0).to(dev)
        X = synthetic.activations(M * self.rotate, K, seed=replica_seed(0, 1, rank), device=dev)
        X[:M] = synthetic.activations(M, K, seed=0).to(dev)
        self.ws = torch.empty(bl.workspace_bytes(bl.BL_OP_W1A8, M, N, K), dtype=torch.uint8, device=dev)
        self.copies = []
        for i in range(self.rotate):
            p, _, b = bl.bin_pack(W[i * N:(i + 1) * N], bl.BL_PACK_BITNET)
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            self.copies.append((X[i * M:(i + 1) * M], p, b, y))
        del W
        self.xh = [self.copies[i][0].cpu().pin_memory() for i in range(16)]
        self.yh = [torch.empty((M, N), dtype=torch.float32).pin_memory() for _ in range(16)]
        self.xd = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        self.yd = torch.empty((M, N), dtype=torch.float32, device=dev)
        self.h2d, self.d2h = 2 * M * K, 4 * M * N

    def step(self, i):
        x, p, b, y = self.copies[i % self.rotate]
        self.bl.bitlinear_w1a8(x, p, b, out=y, ws=self.ws)

    def e2e_step(self, i):
        _, p, b, _ = self.copies[i % self.rotate]
        self.xd.copy_(self.xh[i % 16], non_blocking=True)
        self.bl.bitlinear_w1a8(self.xd, p, b, out=self.yd, ws=self.ws)
        self.yh[i % 16].copy_(self.yd, non_blocking=True)

    def oracle_setup(self):
        import oracle as oracle_pkg
        import synthetic
        self.o = oracle_pkg.get()
        W = synthetic.weights(self.N, self.K, seed=0).numpy()
        self.op, _, self.obeta = self.o.pack_bitnet(W)
        self.ox = synthetic.bf16_bits(synthetic.activations(self.M, self.K, seed=0))
        self.oracle_sample = "the whole M=4, K=N=256 layer per call (single-threaded C oracle, fp64/int64)"
        return float(self.M)

    def oracle_call(self):
        self.o.w1a8(self.ox, self.op, self.obeta, self.K)


class W158A8(W1A8):
    """BitNet b1.58: the W1A8 workload with ternary weights (RoundClip of
    W / mean|W|, two bit planes)."""
    name = "w158a8"
    metric = "BitLinear b1.58 W1.58A8 TOP/s (1.3B shapes, 512 tokens, ternary weights)"
    kernel = "ln_quant_kernel<NV> + gemm_ts_kernel<2,1,T,*> (one call; time includes LN + quantisation)"
    traffic_file = "bitlinear_w158a8_1p3b_512tokens.traffic.json"

    def __init__(self):
        super().__init__()
        self.config = dict(self.config)
        self.config["workload"] = ("BitNet b1.58 BitLinear W1.58A8, 512 tokens, 1.3B shapes 2048->5632 then "
                                   "5632->2048, ternary weights")

    def setup(self, dev, rank):
        import torch
        import bit_linear_layers_b200 as bl
        import synthetic
        self.bl = bl
        self.copies = []
        for i in range(self.rotate):
            layers = []
            for s, (M, K, N) in enumerate(self.SHAPES):
                seed = 4 + 100 * i + 10 * s + 7 * rank
                W = synthetic.weights(N, K, seed=seed, mean=0.001, device=dev)
                p, b = bl.bin_pack(W, bl.BL_PACK_TERNARY)
                del W
                x = synthetic.laplace_channel_activations(M, K, seed=seed, device=dev)
                ws = torch.empty(bl.workspace_bytes(bl.BL_OP_W158A8, M, N, K), dtype=torch.uint8, device=dev)
                y = torch.empty((M, N), dtype=torch.float32, device=dev)
                layers.append((x, p, b, ws, y))
            self.copies.append(layers)
        self.xh = [lay[0].cpu().pin_memory() for lay in self.copies[0]]
        self.yh = [torch.empty_like(lay[4], device="cpu").pin_memory() for lay in self.copies[0]]
        self.h2d = sum(M * K * 2 for M, K, N in self.SHAPES)
        self.d2h = sum(M * N * 4 for M, K, N in self.SHAPES)

    def call(self, x, p, b, ws, y):
        self.bl.bitlinear_w158a8(x, p, b, out=y, ws=ws)

    def oracle_setup(self):
        import oracle as oracle_pkg
        import synthetic
        self.o = oracle_pkg.get()
        self.olayers, ops = [], 0.0
        for s, (M, K, N) in enumerate(self.SHAPES):
            W = synthetic.weights(N, K, seed=4 + 10 * s, mean=0.001).numpy()
            p, gamma_w = self.o.pack_ternary(W)  # gamma needs the whole matrix
            x = synthetic.bf16_bits(synthetic.laplace_channel_activations(1, K, seed=4 + 10 * s))
            self.olayers.append((x, p[:self.ORACLE_COLS].copy(), gamma_w, K))
            ops += 2.0 * K * self.ORACLE_COLS
        self.oracle_sample = ("one token through LN + quantisation and output columns 0..1023 of both "
                              "projections per call, ternary weights (single-threaded C oracle, fp64/int64)")
        return ops

    def oracle_call(self):
        for x, p, gamma_w, K in self.olayers:
            self.o.w158a8(x, p, gamma_w, K)


class W1A8Tensor(W1A8):
    """The W1A8 workload with the per-tensor absmax quantiser (Eq.(5) of the
    "BitNet b1.58" page with gamma over the whole LN output matrix): token
    statistics, one gamma, then quantisation, before the same int8 GEMM. The
    non-negative Eq.(6) form runs the same kernels with one flag."""
    name = "w1a8_tensor"
    metric = "BitLinear W1A8 TOP/s, per-tensor activation gamma (1.3B shapes, 512 tokens)"
    kernel = ("ln_stats_kernel + ln_tensor_scalars_kernel + ln_quant_tensor_kernel + gemm_ts_kernel<1,*> "
              "(one call; time includes LN + quantisation)")
    traffic_file = "bitlinear_w1a8_tensor_1p3b_512tokens.traffic.json"
    launches_per_step = 8

    def __init__(self):
        super().__init__()
        self.config = dict(self.config)
        self.config["workload"] = ("BitNet BitLinear W1A8, 512 tokens, 1.3B shapes 2048->5632 then 5632->2048, "
                                   "per-tensor activation gamma")

    def ws_op(self, bl):
        return bl.BL_OP_W1A8_EX

    def call(self, x, p, b, ws, y):
        self.bl.bitlinear_w1a8_ex(x, p, b, self.bl.BL_W1A8_PER_TENSOR, out=y, ws=ws)

    def oracle_setup(self):
        import oracle as oracle_pkg
        import synthetic
        self.o = oracle_pkg.get()
        self.olayers, ops = [], 0.0
        for s, (M, K, N) in enumerate(self.SHAPES):
            W = synthetic.weights(N, K, seed=4 + 10 * s, mean=0.001).numpy()
            p, _, beta = self.o.pack_bitnet(W)
            x = synthetic.bf16_bits(synthetic.laplace_channel_activations(M, K, seed=4 + 10 * s))
            self.olayers.append((x, p, beta, K))
            ops += 2.0 * K * self.ORACLE_COLS
        self.oracle_sample = ("LN + per-tensor quantisation of all 512 tokens (gamma needs them all), then token 0 "
                              "through output columns 0..1023 of both projections per call (single-threaded C "
                              "oracle, fp64/int64)")
        return ops

    def oracle_call(self):
        import numpy as np
        js = np.arange(self.ORACLE_COLS)
        ms = np.zeros_like(js)
        for x, p, beta, K in self.olayers:
            xq, gamma, _ = self.o.ln_quant_tensor(x, 0)
            acc = self.o.w1a8_acc_at(xq, p, K, ms, js)
            self.o.w1a8_rescale(acc.reshape(1, -1), gamma[:1], beta)


class W1A1(Workload):
    """W1A1 XNOR/popcount products at the 1.3B shapes, 512 tokens, on packed
    +-1 activations and weights. Bound by population-count throughput."""
    name = "w1a1"
    SHAPES = [(512, 2048, 5632), (512, 5632, 2048)]
    metric = "W1A1 XNOR-popcount TOP/s (1.3B shapes, 512 tokens, packed +-1 operands)"
    unit, scale, bound = "TOP/s", 1e12, "alu"
    dtype = "b1"
    kernel = "xnor_gemm_kernel (64x64 tiles, XOR + POPC on the integer pipes)"
    sources = [CSRC + "bl_xnor.cuh", CSRC + "bl_common.cuh", CSRC + "bl_api.cu"]
    traffic_file = "xnor_w1a1_1p3b_512tokens.traffic.json"
    launches_per_step = 2
    rotate = 8
    # 16 population counts per SM per clock (each one 32 +-1 products), 2 ops
    # per product, at the maximum SM clock
    POPC_PER_SM_CLK = 16

    def __init__(self):
        per_copy = sum(M * K // 8 + N * K // 8 + M * N * 4 for M, K, N in self.SHAPES)
        self.config = {"workload": "W1A1 XNOR-popcount products, 512 tokens, 1.3B shapes 2048->5632 then 5632->2048",
                       "shapes_MKN": [list(s) for s in self.SHAPES],
                       "l2": f"{self.rotate} rotating copies ({self.rotate * per_copy / 1e6:.0f} MB); the packed "
                             "operands are small (L2-resident), the int32 outputs stream"}

    def units_per_step(self):
        return sum(2.0 * M * K * N for M, K, N in self.SHAPES)

    def peak(self, peaks, timed_s):
        sms, mhz = 148, 1965.0
        p = sms * self.POPC_PER_SM_CLK * 32 * 2 * mhz * 1e6 / 1e12
        return p, f"derived: {sms} SMs x {self.POPC_PER_SM_CLK} popc/clk x 32 products x 2 ops x {mhz:.0f} MHz"

    def setup(self, dev, rank):
        import torch
        import bit_linear_layers_b200 as bl
        self.bl = bl
        g = torch.Generator(device=dev)
        g.manual_seed(replica_seed(31, 1, rank))
        self.copies = []
        for i in range(self.rotate):
            layers = []
            for (M, K, N) in self.SHAPES:
                a = torch.randint(-2 ** 31, 2 ** 31 - 1, (M, K // 32), generator=g, dtype=torch.int32, device=dev)
                b = torch.randint(-2 ** 31, 2 ** 31 - 1, (N, K // 32), generator=g, dtype=torch.int32, device=dev)
                layers.append((a, b, K, torch.empty((M, N), dtype=torch.int32, device=dev)))
            self.copies.append(layers)
        self.ah = [lay[0].cpu().pin_memory() for lay in self.copies[0]]
        self.yh = [torch.empty_like(lay[3], device="cpu").pin_memory() for lay in self.copies[0]]
        self.h2d = sum(M * K // 8 for M, K, N in self.SHAPES)
        self.d2h = sum(M * N * 4 for M, K, N in self.SHAPES)

    def step(self, i):
        for a, b, K, y in self.copies[i % self.rotate]:
            self.bl.bin_xnor_gemm(a, b, K, out=y)

    def e2e_step(self, i):
        for (a, b, K, y), ah, yh in zip(self.copies[i % self.rotate], self.ah, self.yh):
            a.copy_(ah, non_blocking=True)
            self.bl.bin_xnor_gemm(a, b, K, out=y)
            yh.copy_(y, non_blocking=True)

    ORACLE_COLS = 256

    def oracle_setup(self):
        import numpy as np
        import oracle as oracle_pkg
        self.o = oracle_pkg.get()
        rng = np.random.default_rng(31)
        self.olayers, ops = [], 0.0
        for (M, K, N) in self.SHAPES:
            a = rng.integers(0, 2 ** 32, size=(1, K // 32), dtype=np.uint64).astype(np.uint32)
            b = rng.integers(0, 2 ** 32, size=(self.ORACLE_COLS, K // 32), dtype=np.uint64).astype(np.uint32)
            self.olayers.append((a, b, K))
            ops += 2.0 * K * self.ORACLE_COLS
        self.oracle_sample = ("one packed token against 256 packed rows of both shapes per call "
                              "(single-threaded C oracle, bit by bit)")
        return ops

    def oracle_call(self):
        for a, b, K in self.olayers:
            self.o.w1a1(a, b, K)



_LLAMA7B = {}


def llama7b_layers(dev):
    """The packed signs and scales of all 224 linears of a 7B-shaped model
    (32 layers x q, k, v, o, gate, up, down), built once per process."""
    if dev not in _LLAMA7B:
        import bit_linear_layers_b200 as bl
        import synthetic
        layers = []
        for layer in range(synthetic.LLAMA7B_LAYERS):
            mats = []
            for idx, (K, N) in enumerate(synthetic.LLAMA7B_LAYER):
                W = synthetic.weights(N, K, seed=5000 + 16 * layer + idx, device=dev)
                mats.append(bl.bin_pack(W, bl.BL_PACK_FBI))
                del W
            layers.append(mats)
        _LLAMA7B[dev] = layers
    return _LLAMA7B[dev]


class DecodeStack(Workload):
    """Decode of a 7B-shaped FBI-LLM's linears (32 layers x q, k, v, o,
    gate, up, down; 0.8 GB of packed signs, more than L2) at batch B, one
    bin_linear_w1a16_stack(_batch) call per token step: 128 levels per
    step (q, k, v from the layer input; o from v; gate, up from o; down
    from up, which feeds the next layer), every linear writing a buffer of
    its own. A step is one token step of all B tokens through all 224
    linears."""
    name = "decode_stack"
    B = 1
    metric = ("7B-shaped FBI-LLM linear-only decode tok/s at batch 1 (W1A16, 32 layers x 7 linears, "
              "one stacked call per token step)")
    unit, scale, bound = "tok/s", 1.0, "hbm"
    roof_unit = "GB/s"
    kernel = ("gemv_w1a16_stream_kernel (15 clusters of 8 CTAs, persistent; two launches per step: 82 + 46 "
              "levels, at most 144 linears per launch)")
    sources = [CSRC + "bl_gemv_stream.cuh", CSRC + "bl_gemv_lut.cuh", CSRC + "bl_common.cuh", CSRC + "bl_api.cu"]
    traffic_file = "gemv_w1a16_stream_7b_decode_batch1.traffic.json"
    traffic_per = "step"  # achieved and traffic both cover the step's two launches
    launches_per_step = 2

    def __init__(self):
        import synthetic
        B = self.B
        self.linears = [(K, N) for _ in range(synthetic.LLAMA7B_LAYERS) for K, N in synthetic.LLAMA7B_LAYER]
        self.packed_b = sum(N * K // 8 for K, N in self.linears)
        self.alg_b = sum(N * K // 8 + 4 * N + 2 * B * K + 2 * B * N for K, N in self.linears)
        self.config = {"workload": f"all 224 linears of a 7B-shaped FBI-LLM (32 layers x q,k,v,o 4096x4096; gate,up "
                                   f"4096->11008; down 11008->4096), W1A16 decode at batch {B}",
                       "batch": B, "layers": synthetic.LLAMA7B_LAYERS, "levels_per_step": 4 * synthetic.LLAMA7B_LAYERS,
                       "packed_bytes_per_step": self.packed_b, "algorithmic_bytes_per_step": self.alg_b,
                       "l2": f"inputs larger than L2: {self.packed_b / 1e6:.0f} MB of packed signs streamed per step",
                       "call": "bin_linear_w1a16_stack" + ("" if B == 1 else "_batch") +
                               " (a zero-fill of the tagged outputs, then one persistent launch per 96 levels "
                               "or 144 linears)"}

    def units_per_step(self):
        return float(self.B)  # tokens

    def achieved(self, per_step_s):
        return self.alg_b / per_step_s / 1e9  # all bytes the step must move

    def peak(self, peaks, timed_s):
        return peaks["hbm_gbs"], "hbm_gbs"

    def setup(self, dev, rank):
        import torch
        import bit_linear_layers_b200 as bl
        import synthetic
        B = self.B
        layers = llama7b_layers(dev)
        shp = (lambda n: (n,)) if B == 1 else (lambda n: (B, n))
        self.x = synthetic.activations(B, 4096, seed=77 + 7 * rank, device=dev).reshape(shp(4096))
        levels, cur = [], self.x
        for mats in layers:
            q, k, v, o, h = (torch.empty(shp(4096), dtype=torch.bfloat16, device=dev) for _ in range(5))
            g, u = (torch.empty(shp(11008), dtype=torch.bfloat16, device=dev) for _ in range(2))
            levels.append((cur, [(mats[0][0], mats[0][1], q), (mats[1][0], mats[1][1], k),
                                 (mats[2][0], mats[2][1], v)]))
            levels.append((v, [(mats[3][0], mats[3][1], o)]))
            levels.append((o, [(mats[4][0], mats[4][1], g), (mats[5][0], mats[5][1], u)]))
            levels.append((u, [(mats[6][0], mats[6][1], h)]))
            cur = h
        self.h = cur
        self.stack = bl.W1A16Stack(levels)
        self.xh = [self.x.cpu().pin_memory() for _ in range(2)]
        self.hh = [torch.empty_like(self.h, device="cpu").pin_memory() for _ in range(2)]
        self.h2d, self.d2h = 2 * B * 4096, 2 * B * 4096

    def step(self, i):
        self.stack.run()

    def e2e_step(self, i):
        self.x.copy_(self.xh[i % 2], non_blocking=True)
        self.stack.run()
        self.hh[i % 2].copy_(self.h, non_blocking=True)

    # oracle: output rows [0, 256) of each linear of layer 0, all B tokens, per call
    ORACLE_ROWS = 256

    def oracle_setup(self):
        import oracle as oracle_pkg
        import synthetic
        self.o = oracle_pkg.get()
        self.olin, work = [], 0.0
        for idx, (K, N) in enumerate(synthetic.LLAMA7B_LAYER):
            W = synthetic.weights(self.ORACLE_ROWS, K, seed=5000 + idx).numpy()
            packed, alpha = self.o.pack_fbi(W)
            x = synthetic.bf16_bits(synthetic.activations(self.B, K, seed=77 + idx))
            self.olin.append((x, packed, alpha, K))
            work += self.ORACLE_ROWS * K
        self.oracle_sample = (f"output rows 0..{self.ORACLE_ROWS - 1} of each of the 7 linear shapes of a layer for "
                              f"{self.B} token(s) per call (single-threaded C oracle, fp64)")
        return self.B * work / sum(N * K for K, N in self.linears)  # token steps per call

    def oracle_call(self):
        for x, packed, alpha, K in self.olin:
            self.o.w1a16(x, packed, alpha, K)


class DecodeStack16(DecodeStack):
    name = "decode_stack16"
    B = 16
    metric = ("7B-shaped FBI-LLM linear-only decode tok/s at batch 16 (W1A16, 32 layers x 7 linears, "
              "one stacked call per token step)")
    kernel = ("gemv_w1a16_stream_mma_kernel<16> (15 clusters of 8 CTAs, persistent; two launches per step: "
              "82 + 46 levels, at most 144 linears per launch)")
    sources = [CSRC + "bl_gemv_stream_mma.cuh", CSRC + "bl_gemv_stream.cuh", CSRC + "bl_gemv_mma.cuh",
               CSRC + "bl_common.cuh", CSRC + "bl_api.cu"]
    traffic_file = "gemv_w1a16_stream_mma_7b_decode_batch16.traffic.json"


WORKLOADS = {w.name: w for w in (Decode, Prefill, Backward, W1A8, W1A8Single, W158A8, W1A8Tensor, W1A1,
                                   DecodeStack, DecodeStack16)}


# ----------------------------------------------------------------------------- ours


def _capture(step, first, count, stream):
    """A CUDA graph of `count` steps whose first and last nodes record two
    timing events (external event nodes), so that the events bracket exactly
    the steps' device work and not the graph's own launch."""
    import torch
    graph = torch.cuda.CUDAGraph()
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            e0.record(stream)
            for i in range(count):
                step(first + i)
            e1.record(stream)
    torch.cuda.synchronize()
    graph.replay()  # untimed replay: the graph's first launch uploads it
    torch.cuda.synchronize()
    return graph, (e0, e1)


def _timed_replay(captured, dev, world):
    import torch
    graph, (e0, e1) = captured
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    return e0.elapsed_time(e1)


def run_workload(wl, steps, warmup, rank, world, dev, sampler=None):
    """Device-resident and end-to-end times (ms) of `steps` steps, max over ranks."""
    import torch
    wl.setup(dev, rank)
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.start()
    # settle clocks (untimed, about a second), then exactly W warm-up steps
    t_end, i = time.time() + 1.0, 0
    while time.time() < t_end:
        for _ in range(max(1, 256 // wl.launches_per_step)):
            wl.step(i)
            i += 1
        torch.cuda.synchronize()
    for i in range(warmup):
        wl.step(i)
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream(dev))
    graph = _capture(wl.step, warmup, steps, stream)
    ms = _timed_replay(graph, dev, world)
    del graph

    for i in range(warmup):
        wl.e2e_step(i)
    torch.cuda.synchronize()
    g2 = _capture(wl.e2e_step, warmup, steps, stream)
    ms_e2e = _timed_replay(g2, dev, world)
    del g2
    clocks = sampler.stop() if sampler is not None else None

    ms, ms_e2e = max_over_ranks([ms, ms_e2e], world, dev)
    return ms, ms_e2e, clocks


def max_over_ranks(times, world, device):
    """Each rank's device-timed milliseconds -> the maximum over all ranks
    (every rank takes part; a no-op for one rank)."""
    if world <= 1:
        return list(times)
    import torch
    t = torch.tensor(times, dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t]


def replica_seed(base, copy, rank):
    """Seed of rotating input copy `copy` on `rank`: copy 0 is the seeded
    workload itself on every rank; the others differ per rank, so replicas
    do not stream identical weights."""
    return base if copy == 0 else base + 1000 * copy + 7 * rank


def whole_job_value(world, steps, units_per_step, ms, scale):
    """Aggregate throughput of all ranks: every rank processed `steps`
    steps of `units_per_step` units in at most `ms` milliseconds."""
    return world * steps * units_per_step / (ms * 1e-3) / scale


def cpu_baseline(wl, target_s=10.0):
    """The oracle as it stands, on the host, over repeated bounded samples."""
    units = wl.oracle_setup()
    reps, t0 = 0, time.perf_counter()
    while True:
        wl.oracle_call()
        reps += 1
        el = time.perf_counter() - t0
        if el >= target_s:
            break
    return {"value": reps * units / el / wl.scale, "unit": wl.unit, "cores": 1, "kind": "oracle",
            "sample": f"{wl.oracle_sample}; {reps} calls in {el:.1f} s"}


def summarize(wl, ms, ms_e2e, steps, world, peaks, peak_kind):
    per_step_s = ms * 1e-3 / steps
    timed_s = ms * 1e-3
    peak, peak_key = wl.peak(peaks, timed_s)
    achieved = wl.achieved(per_step_s)
    roof = {"bound": wl.bound, "achieved": achieved, "peak": peak, "unit": getattr(wl, "roof_unit", wl.unit),
            "frac": achieved / peak, "traffic": wl.traffic(), "traffic_per": getattr(wl, "traffic_per", "launch"),
            "kernel": wl.kernel,
            "peak_source": peak_key if peak_key.startswith("derived")
            else (f"{peak_kind}: MEASURED_PEAKS.json {peak_key}" if peak_kind == "measured" else f"fallback ({peak_key})")}
    if isinstance(wl, Decode):
        roof["algorithmic_bytes_per_launch"] = wl.alg_b
    value = whole_job_value(world, steps, wl.units_per_step(), ms, wl.scale)
    e2e = {"value": whole_job_value(world, steps, wl.units_per_step(), ms_e2e, wl.scale), "unit": wl.unit,
           "h2d_bytes_per_step": wl.h2d, "d2h_bytes_per_step": wl.d2h, "ms_per_step": ms_e2e / steps}
    return value, roof, e2e


def secondary_llama7b(dev, peaks):
    """All 224 linears of a 7B-shaped model (0.8 GB of signs, more than L2):
    decode at batch 1 and 16 as a chain of 224 launches per token step
    (x -> q,k,v; v -> o; o -> gate,up; up -> down -> next layer), CUDA graph
    of one step, and a 4096-token prefill. The same chain as one stacked
    call per step is the decode_stack / decode_stack16 workload."""
    import torch
    import bit_linear_layers_b200 as bl
    import synthetic
    layers = llama7b_layers(dev)
    packed_bytes = sum(p.numel() * 4 for mats in layers for p, _ in mats)
    flags = bl.BL_FLAG_OVERLAP_PREVIOUS
    res = {"packed_GB": packed_bytes / 1e9}
    for B in (1, 16):
        x = synthetic.activations(B, 4096, seed=77, device=dev)
        q, k, v, o = (torch.empty((B, 4096), dtype=torch.bfloat16, device=dev) for _ in range(4))
        g, u = (torch.empty((B, 11008), dtype=torch.bfloat16, device=dev) for _ in range(2))
        h = torch.empty((B, 4096), dtype=torch.bfloat16, device=dev)

        def step():
            cur = x
            for mats in layers:
                bl.bin_linear_w1a16(cur, *mats[0], out=q, flags=flags)
                bl.bin_linear_w1a16(cur, *mats[1], out=k, flags=flags)
                bl.bin_linear_w1a16(cur, *mats[2], out=v, flags=flags)
                bl.bin_linear_w1a16(v, *mats[3], out=o, flags=flags)
                bl.bin_linear_w1a16(o, *mats[4], out=g, flags=flags)
                bl.bin_linear_w1a16(o, *mats[5], out=u, flags=flags)
                bl.bin_linear_w1a16(u, *mats[6], out=h, flags=flags)
                cur = h

        for _ in range(3):
            step()
        torch.cuda.synchronize()
        gph = torch.cuda.CUDAGraph()
        st = torch.cuda.Stream(device=dev)
        st.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(st):
            with torch.cuda.graph(gph, stream=st):
                step()
        gph.replay()
        torch.cuda.synchronize()
        reps = 20
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            gph.replay()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        res[f"decode_batch{B}"] = {"ms_per_token_step": ms, "tok_s": B / (ms * 1e-3),
                                   "packed_GB_per_s": packed_bytes / (ms * 1e-3) / 1e9,
                                   "hbm_frac": packed_bytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                   "launches_per_step": 224}
        del gph
    # prefill: 4096 tokens through every linear (not chained: fixed inputs)
    T = 4096
    x4 = synthetic.activations(T, 4096, seed=78, device=dev)
    x11 = synthetic.activations(T, 11008, seed=79, device=dev)
    y4 = torch.empty((T, 4096), dtype=torch.bfloat16, device=dev)
    y11 = torch.empty((T, 11008), dtype=torch.bfloat16, device=dev)

    def prefill():
        for mats in layers:
            for idx, (K, N) in enumerate(synthetic.LLAMA7B_LAYER):
                bl.bin_linear_w1a16(x4 if K == 4096 else x11, *mats[idx], out=y4 if N == 4096 else y11)

    prefill()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    prefill()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    flop = sum(2.0 * T * K * N for (K, N) in synthetic.LLAMA7B_LAYER) * synthetic.LLAMA7B_LAYERS
    res["prefill_4096"] = {"ms": ms, "tok_s": T / (ms * 1e-3), "tflops": flop / (ms * 1e-3) / 1e12,
                           "tensor_frac": flop / (ms * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"],
                           "peak_source": "measured bf16 sustained (a long step)"}
    res["metric"] = "linear-only tokens/s of a 7B-shaped FBI-LLM (32 layers x 7 linears)"
    return res


def secondary(args, dev, peaks, peak_kind):
    """The workloads other than the headline one, 200 steps each, plus the
    7B-shaped model. Only at N=1."""
    import gc
    import torch
    out = {}
    for name, cls in WORKLOADS.items():
        if name == args.workload:
            continue
        wl = cls()
        steps = 200
        ms, ms_e2e, _ = run_workload(wl, steps, 3, 0, 1, dev)
        value, roof, e2e = summarize(wl, ms, ms_e2e, steps, 1, peaks, peak_kind)
        out[name] = {"metric": wl.metric, "value": value, "unit": wl.unit, "ms_per_step": ms / steps,
                     "steps": steps, "warmup": 3, "config": wl.config, "roofline": roof, "e2e": e2e,
                     "gpu_launches": steps * wl.launches_per_step}
        del wl
        gc.collect()
        torch.cuda.empty_cache()
    out["pack"] = secondary_pack(dev, peaks)
    out["few_tokens"] = secondary_few_tokens(dev, peaks)
    out["decode_l2_warm"] = secondary_decode_warm(dev)
    out["llama7b_linear"] = secondary_llama7b(dev, peaks)
    return out


def secondary_few_tokens(dev, peaks):
    """The few-token paths at decode shapes, each timed as a graph of launches
    over rotating copies (more than L2): W1A16 at 2..16 tokens on 4096x4096
    (the 7B attention projection) and W1A8 at 1..16 tokens on 2048->5632 (the
    1.3B MLP up-projection); GB/s counts the bytes a call must move."""
    import torch
    import bit_linear_layers_b200 as bl
    import synthetic
    res = {"l2": "rotating copies larger than L2; one CUDA graph of 400 calls, CUDA events"}
    calls = 400

    def time_graph(fn, n):
        st = torch.cuda.Stream(device=dev)
        st.wait_stream(torch.cuda.current_stream(dev))
        for i in range(8):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(st):
            with torch.cuda.graph(g, stream=st):
                for i in range(n):
                    fn(i)
        g.replay()
        torch.cuda.synchronize()
        ms = _median_ms(g.replay, reps=5)
        del g
        return ms / n

    K = N = 4096
    copies = 64  # 2 MB of signs each
    packs = []
    for i in range(copies):
        W = synthetic.weights(N, K, seed=3000 + i, device=dev)
        packs.append(bl.bin_pack(W, bl.BL_PACK_FBI))
        del W
    for M in (2, 4, 8, 16):
        xs = [synthetic.activations(M, K, seed=3100 + i, device=dev) for i in range(copies)]
        ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(copies)]

        def fn(i, xs=xs, ys=ys):
            j = i % copies
            bl.bin_linear_w1a16(xs[j], *packs[j], out=ys[j], flags=bl.BL_FLAG_OVERLAP_PREVIOUS)

        s_call = time_graph(fn, calls) * 1e-3
        nbytes = N * K // 8 + 4 * N + 2 * M * K + 2 * M * N
        res[f"w1a16_M{M}_4096x4096"] = {"us_per_call": s_call * 1e6, "GB_s": nbytes / s_call / 1e9,
                                        "hbm_frac": nbytes / s_call / 1e9 / peaks["hbm_gbs"]}
    del packs
    K, N = 2048, 5632
    copies = 96  # 1.4 MB of signs each
    layers = []
    for i in range(copies):
        W = synthetic.weights(N, K, seed=3200 + i, mean=0.001, device=dev)
        p, _, b = bl.bin_pack(W, bl.BL_PACK_BITNET)
        layers.append((p, b))
        del W
    for M in (1, 4, 16):
        xs = [synthetic.laplace_channel_activations(M, K, seed=3300 + i, device=dev) for i in range(copies)]
        ys = [torch.empty((M, N), dtype=torch.float32, device=dev) for _ in range(copies)]
        ws = torch.empty(bl.workspace_bytes(bl.BL_OP_W1A8, M, N, K), dtype=torch.uint8, device=dev)

        def fn(i, xs=xs, ys=ys, ws=ws):
            j = i % copies
            bl.bitlinear_w1a8(xs[j], *layers[j], out=ys[j], ws=ws)

        s_call = time_graph(fn, calls) * 1e-3
        nbytes = N * K // 8 + 2 * M * K + 4 * M * N
        res[f"w1a8_M{M}_2048x5632"] = {"us_per_call": s_call * 1e6, "GB_s": nbytes / s_call / 1e9,
                                       "hbm_frac": nbytes / s_call / 1e9 / peaks["hbm_gbs"],
                                       "launches": 2}
    return res


def secondary_pack(dev, peaks):
    """bin_pack of a 4096 x 11008 fp32 matrix (180 MB, more than L2) in both
    modes: GB/s on the bytes it must move (W read, packed bits and scales written)."""
    import torch
    import bit_linear_layers_b200 as bl
    import synthetic
    N, K = 11008, 4096
    W = synthetic.weights(N, K, seed=6, device=dev)
    res = {}
    for mode, name in ((bl.BL_PACK_FBI, "fbi"), (bl.BL_PACK_BITNET, "bitnet")):
        packed = torch.empty((N, K // 32), dtype=torch.int32, device=dev)
        alpha = torch.empty(N if mode == bl.BL_PACK_FBI else 1, dtype=torch.float32, device=dev)
        beta = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.empty(max(1, bl.workspace_bytes(bl.BL_OP_PACK_BITNET if mode else bl.BL_OP_PACK_FBI, 0, N, K)),
                         dtype=torch.uint8, device=dev)

        def call():
            bl.bin_pack(W, mode, packed=packed, alpha=alpha, beta=beta, ws=ws)

        ms = _median_ms(call, reps=10)
        nbytes = 4 * N * K + N * K // 8 + 4 * alpha.numel()
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[name] = {"shape_NK": [N, K], "us": ms * 1e3, "GB_s": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
                     "launches": 1 if mode == bl.BL_PACK_FBI else 3}
    res["l2"] = "W is 180 MB, more than L2"
    return res


def secondary_decode_warm(dev):
    """Single-launch latency of the decode GEMV with no rotation (weights
    L2-warm), one launch per step in a CUDA graph, with and without
    programmatic dependent launch."""
    import torch
    import bit_linear_layers_b200 as bl
    import synthetic
    W = synthetic.weights(4096, 4096, seed=2, device=dev)
    p, a = bl.bin_pack(W, bl.BL_PACK_FBI)
    x = synthetic.activations(1, 4096, seed=2, device=dev)
    y = torch.empty((1, 4096), dtype=torch.bfloat16, device=dev)
    res = {"label": "L2-warm: the same 2 MB of weights every launch"}
    for flags, name in ((0, "plain"), (bl.BL_FLAG_OVERLAP_PREVIOUS, "overlap_previous")):
        reps = 200
        st = torch.cuda.Stream(device=dev)
        st.wait_stream(torch.cuda.current_stream(dev))
        for _ in range(5):
            bl.bin_linear_w1a16(x, p, a, out=y, flags=flags)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(st):
            with torch.cuda.graph(g, stream=st):
                for _ in range(reps):
                    bl.bin_linear_w1a16(x, p, a, out=y, flags=flags)
        g.replay()
        torch.cuda.synchronize()
        res[f"{name}_us_per_launch"] = _median_ms(g.replay, reps=5) * 1e3 / reps
        del g
    return res


def _median_ms(fn, reps=5):
    import torch
    fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    ts.sort()
    return ts[len(ts) // 2]


# ----------------------------------------------------------------------------- main


def probe_int8(dev):
    """Dense int8 GEMM throughput of a library kernel (torch._int_mm, s8 x s8
    -> s32, M = N = K = 8192): best of 10 launches and the mean of a 2 s loop,
    in TOP/s (2 MNK per product). A reference point for the W1A8 rooflines."""
    import torch
    n = 8192
    a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
    b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev).t().contiguous().t()
    for _ in range(3):
        torch._int_mm(a, b)
    torch.cuda.synchronize()
    best = min(_median_ms(lambda: torch._int_mm(a, b), reps=1) for _ in range(10))
    reps, t_end = 0, time.time() + 2.0
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    while time.time() < t_end:
        for _ in range(20):
            torch._int_mm(a, b)
        reps += 20
    e1.record()
    torch.cuda.synchronize()
    sustained = e0.elapsed_time(e1) / reps
    ops = 2.0 * n ** 3
    return {"probe": "torch._int_mm s8 x s8 -> s32, 8192^3", "burst_tops": ops / (best * 1e-3) / 1e12,
            "sustained_tops": ops / (sustained * 1e-3) / 1e12, "best_ms": best, "sustained_ms": sustained,
            "gpu": torch.cuda.get_device_name(dev)}


def main():
    args = parse()
    if args.probe_int8:
        import torch
        dev = torch.device("cuda", 0)
        sampler = ClockSampler(0)
        sampler.start()
        res = probe_int8(dev)
        res["clocks"] = sampler.stop()
        print(json.dumps(res), flush=True)
        return 0
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = WORKLOADS[args.workload]()
    wl_metric, wl_unit, wl_dtype, wl_launches = wl.metric, wl.unit, wl.dtype, wl.launches_per_step
    config = dict(wl.config)
    config["timing"] = ("K steps in one CUDA graph, timed by CUDA events recorded as the graph's first and last "
                        "nodes (the launching stream)")
    config["parallelism"] = f"replicas x{world}"

    if args.impl == "reference":
        if rank != 0:
            return 0
        units = wl.oracle_setup()
        for _ in range(args.warmup):
            wl.oracle_call()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            wl.oracle_call()
        el = time.perf_counter() - t0
        value = args.steps * units / el / wl.scale
        line = {"impl": "reference", "metric": wl.metric, "value": value, "unit": wl.unit, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config,
                "cpu_baseline": {"value": value, "unit": wl.unit, "cores": 1, "kind": "oracle",
                                 "sample": f"{wl.oracle_sample}; one call per step"},
                "e2e": {"value": value, "unit": wl.unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    visible = [v for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    sampler = ClockSampler(visible[local_rank] if local_rank < len(visible) else local_rank)
    ms, ms_e2e, clocks = run_workload(wl, args.steps, args.warmup, rank, world, dev, sampler)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0
    peaks, peak_kind = load_peaks()
    value, roof, e2e = summarize(wl, ms, ms_e2e, args.steps, world, peaks, peak_kind)
    cpu = cpu_baseline(wl) if world == 1 else None
    extra = None
    if world == 1 and not args.no_secondary:
        del wl
        torch.cuda.empty_cache()
        extra = secondary(args, dev, peaks, peak_kind)
    line = {
        "metric": wl_metric, "value": value, "unit": wl_unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl_dtype, "data": "synthetic",
        "config": config, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": args.steps * wl_launches,
        "clocks": clocks, "secondary": extra,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
