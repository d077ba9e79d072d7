#!/usr/bin/env python
"""Benchmark of the binarized linear layers on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Default workload: the FBI-linear W1A16 decode GEMV, M=1 token, K=N=4096
(a 7B attention projection), judged on packed-weight bytes per second. A
step is one call of the layer on one token. Between steps the weights
rotate over 128 distinct packed copies (268 MB, more than twice the 126 MB
L2), so every step streams its weights from HBM. After W untimed warm-up
steps, K steps are captured in one CUDA graph and timed with CUDA events on
the launching stream; with N ranks (torchrun) every rank runs its own
replica (no data-path collective) and the time is the max over ranks.

Rank 0 prints one JSON line. `--impl reference` times the CPU oracle on the
same workload instead (the reference arm of this benchmark).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
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
M_DEC, K_DEC, N_DEC = 1, 4096, 4096
ROTATE = 128
KERNEL_SOURCES = ["bit_linear_layers_b200/csrc/bl_gemv_lut.cuh", "bit_linear_layers_b200/csrc/bl_common.cuh",
                  "bit_linear_layers_b200/csrc/bl_api.cu"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gemv_w1a16_decode_1x4096x4096.traffic.json")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
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


def kernel_src_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_per_launch():
    """DRAM bytes per launch from the committed ncu summary, or None when the
    summary is missing or was taken on a different version of the kernel."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    if d.get("src_hash") != kernel_src_hash():
        return None
    return d.get("dram_bytes_per_launch")


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


# ----------------------------------------------------------------------------- ours


def run_ours(args, rank, world, local_rank):
    import torch
    import bit_linear_layers_b200 as bl
    from bit_linear_layers_b200 import synthetic

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    M, K, N = M_DEC, K_DEC, N_DEC
    # weights: copy 0 is the seeded workload (CPU generator), the others are
    # further seeded draws made on the device
    packs, alphas, xs = [], [], []
    for i in range(ROTATE):
        if i == 0:
            W = synthetic.weights(N, K, seed=2).to(dev)
            x = synthetic.activations(M, K, seed=2).to(dev)
        else:
            W = synthetic.weights(N, K, seed=2 + 1000 * i + 7 * rank, device=dev)
            x = synthetic.activations(M, K, seed=2 + 1000 * i + 7 * rank, device=dev)
        p, a = bl.bin_pack(W, bl.BL_PACK_FBI)
        packs.append(p)
        alphas.append(a)
        xs.append(x)
        del W
    ys = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(ROTATE)]
    torch.cuda.synchronize()

    # consecutive steps never write each other's weights, so each launch may
    # start streaming its weights while the previous one finishes
    flags = bl.BL_FLAG_OVERLAP_PREVIOUS

    def step(i):
        j = i % ROTATE
        bl.bin_linear_w1a16(xs[j], packs[j], alphas[j], out=ys[j], flags=flags)

    visible = [v for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    sampler = ClockSampler(visible[local_rank] if local_rank < len(visible) else local_rank)
    sampler.start()
    # settle clocks (untimed), then exactly W warm-up steps
    t_end = time.time() + 1.0
    while time.time() < t_end:
        for i in range(256):
            step(i)
        torch.cuda.synchronize()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    K_steps = args.steps
    graph = torch.cuda.CUDAGraph()
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            for i in range(K_steps):
                step(args.warmup + i)
    torch.cuda.synchronize()
    graph.replay()  # untimed replay: the graph's first launch uploads it
    torch.cuda.synchronize()

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    launch_stream = torch.cuda.current_stream(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(launch_stream)
    graph.replay()
    e1.record(launch_stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = e0.elapsed_time(e1)

    # end to end through host buffers: x from pinned host, y back to pinned host
    xh = [x.cpu().pin_memory() for x in xs]
    yh = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(ROTATE)]
    xd = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    yd = torch.empty((M, N), dtype=torch.bfloat16, device=dev)

    def e2e_step(i):
        j = i % ROTATE
        xd.copy_(xh[j], non_blocking=True)
        bl.bin_linear_w1a16(xd, packs[j], alphas[j], out=yd, flags=flags)
        yh[j].copy_(yd, non_blocking=True)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g2, stream=stream):
            for i in range(K_steps):
                e2e_step(i)
    g2.replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0.record(launch_stream)
    g2.replay()
    e1.record(launch_stream)
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1)
    clocks = sampler.stop()

    if world > 1:
        t = torch.tensor([ms, ms_e2e], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms, ms_e2e = float(t[0]), float(t[1])
    del graph, g2
    return ms, ms_e2e, clocks


def cpu_baseline_decode(target_s=10.0, cap_s=30.0):
    import numpy as np
    import oracle as oracle_pkg
    from bit_linear_layers_b200 import synthetic

    o = oracle_pkg.get()
    W = synthetic.weights(N_DEC, K_DEC, seed=2).numpy()
    x = synthetic.bf16_bits(synthetic.activations(M_DEC, K_DEC, seed=2))
    packed, alpha = o.pack_fbi(W)
    reps, t0 = 0, time.perf_counter()
    while True:
        o.w1a16(x, packed, alpha, K_DEC)
        reps += 1
        el = time.perf_counter() - t0
        if el >= target_s or el >= cap_s:
            break
    gbs = reps * (N_DEC * K_DEC / 8) / el / 1e9
    return {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"the full 1x4096x4096 decode problem, {reps} calls in {el:.1f} s "
                      "(single-threaded C oracle, fp64)"}, np


def bytes_per_step():
    packed = N_DEC * K_DEC // 8
    alg = packed + 4 * N_DEC + 2 * M_DEC * K_DEC + 2 * M_DEC * N_DEC
    return packed, alg


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    packed_b, alg_b = bytes_per_step()
    metric = "decode GEMV HBM GB/s on packed-weight bytes (W1A16, 1x4096x4096)"
    config = {"workload": "FBI-linear W1A16 decode GEMV, M=1, K=4096, N=4096 (7B attention projection)",
              "M": M_DEC, "K": K_DEC, "N": N_DEC,
              "l2": f"inputs larger than L2: {ROTATE} distinct packed weight copies "
                    f"({ROTATE * packed_b / 1e6:.0f} MB) rotated step to step",
              "timing": "K steps in one CUDA graph, CUDA events on the launching stream",
              "launch": "programmatic dependent launch between steps (BL_FLAG_OVERLAP_PREVIOUS)",
              "parallelism": f"replicas x{world}"}

    if args.impl == "reference":
        if rank != 0:
            return 0
        import oracle as oracle_pkg
        from bit_linear_layers_b200 import synthetic
        o = oracle_pkg.get()
        W = synthetic.weights(N_DEC, K_DEC, seed=2).numpy()
        x = synthetic.bf16_bits(synthetic.activations(M_DEC, K_DEC, seed=2))
        packed, alpha = o.pack_fbi(W)
        for _ in range(args.warmup):
            o.w1a16(x, packed, alpha, K_DEC)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            o.w1a16(x, packed, alpha, K_DEC)
        el = time.perf_counter() - t0
        value = args.steps * packed_b / el / 1e9
        line = {"impl": "reference", "metric": metric, "value": value, "unit": "GB/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config,
                "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                 "sample": f"the full decode problem once per step, {args.steps} steps"},
                "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    ms, ms_e2e, clocks = run_ours(args, rank, world, local_rank)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0
    peaks, peak_kind = load_peaks()
    per_step_ms = ms / args.steps
    value = world * args.steps * packed_b / (ms * 1e-3) / 1e9
    achieved = alg_b / (per_step_ms * 1e-3) / 1e9
    cpu, _ = cpu_baseline_decode()
    line = {
        "metric": metric, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": per_step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic_per_launch(),
                     "kernel": "gemv_w1a16_lut_kernel<1> (cluster of 8 x 16 clusters)", "algorithmic_bytes_per_launch": alg_b,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                     else "fallback 6.65 TB/s"},
        "cpu_baseline": cpu,
        "e2e": {"value": world * args.steps * packed_b / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": 2 * M_DEC * K_DEC, "d2h_bytes_per_step": 2 * M_DEC * N_DEC,
                "ms_per_step": ms_e2e / args.steps},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
