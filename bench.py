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
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the prefill, W1A8 and 7B measurements that ride along at N=1")
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


# ----------------------------------------------------------------------------- secondary

def _flush_buffer(dev):
    import torch
    return torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # 256 MB > 126 MB L2


def _timed_call(fn, flush, reps=5):
    """Median device time (ms) of fn() with L2 flushed before every call."""
    import torch
    ts = []
    for _ in range(2):
        fn()
    for _ in range(reps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    ts.sort()
    return ts[len(ts) // 2]


def secondary_prefill(dev, peaks, flush):
    """W1A16 prefill on the 7B MLP shapes: TFLOPS vs the measured bf16 peak."""
    import bit_linear_layers_b200 as bl
    from bit_linear_layers_b200 import synthetic
    out, total_flop, total_ms = [], 0.0, 0.0
    for (M, K, N) in [(2048, 4096, 11008), (2048, 11008, 4096)]:
        W = synthetic.weights(N, K, seed=1, device=dev)
        x = synthetic.activations(M, K, seed=1, device=dev)
        p, a = bl.bin_pack(W, bl.BL_PACK_FBI)
        del W
        ms = _timed_call(lambda: bl.bin_linear_w1a16(x, p, a), flush)
        flop = 2.0 * M * N * K
        out.append({"shape": f"{M}x{K}x{N}", "us": ms * 1e3, "tflops": flop / (ms * 1e-3) / 1e12})
        total_flop += flop
        total_ms += ms
    tf = total_flop / (total_ms * 1e-3) / 1e12
    return {"metric": "prefill TFLOPS (W1A16, 7B MLP shapes, 2048 tokens)", "tflops": tf,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tf / peaks["bf16_tflops"], "kernel": "gemm_ts_kernel<0,128>",
                         "peak_source": "measured bf16 burst (MEASURED_PEAKS.json bf16_tflops)"},
            "shapes": out, "l2": "flushed (256 MB write) before every call"}


def secondary_w1a8(dev, peaks, flush):
    """BitLinear W1A8 at the 1.3B shapes (512 tokens): LN+quant and int8 GEMM."""
    import torch
    import bit_linear_layers_b200 as bl
    from bit_linear_layers_b200 import synthetic
    int8_peak = 2.0 * peaks["bf16_tflops"]
    out, total_op, total_ms = [], 0.0, 0.0
    for (M, K, N) in [(512, 2048, 5632), (512, 5632, 2048)]:
        W = synthetic.weights(N, K, seed=4, mean=0.001, device=dev)
        x = synthetic.laplace_channel_activations(M, K, seed=4, device=dev)
        p, _, b = bl.bin_pack(W, bl.BL_PACK_BITNET)
        del W
        ws = torch.empty(bl.workspace_bytes(bl.BL_OP_W1A8, M, N, K), dtype=torch.uint8, device=dev)
        y = torch.empty((M, N), dtype=torch.float32, device=dev)
        ms = _timed_call(lambda: bl.bitlinear_w1a8(x, p, b, out=y, ws=ws), flush)
        op = 2.0 * M * N * K
        out.append({"shape": f"{M}x{K}x{N}", "us": ms * 1e3, "tops": op / (ms * 1e-3) / 1e12})
        total_op += op
        total_ms += ms
    tops = total_op / (total_ms * 1e-3) / 1e12
    return {"metric": "BitLinear W1A8 TOPS (1.3B shapes, 512 tokens, LN + quant + int8 GEMM)", "tops": tops,
            "roofline": {"bound": "tensor", "achieved": tops, "peak": int8_peak, "unit": "TOP/s",
                         "frac": tops / int8_peak,
                         "peak_source": "measured bf16 burst x nominal int8/bf16 ratio 2"},
            "shapes": out, "l2": "flushed (256 MB write) before every call"}


def secondary_llama7b(dev, peaks):
    """All 224 linears of a 7B-shaped model (0.8 GB of signs, more than L2):
    decode at batch 1 and 16 as one dependent chain per token step
    (x -> q,k,v; v -> o; o -> gate,up; up -> down -> next layer), CUDA graph
    of one step, and a 4096-token prefill."""
    import torch
    import bit_linear_layers_b200 as bl
    from bit_linear_layers_b200 import synthetic
    layers = []
    for layer in range(synthetic.LLAMA7B_LAYERS):
        mats = []
        for idx, (K, N) in enumerate(synthetic.LLAMA7B_LAYER):
            W = synthetic.weights(N, K, seed=5000 + 16 * layer + idx, device=dev)
            mats.append(bl.bin_pack(W, bl.BL_PACK_FBI))
            del W
        layers.append(mats)
    packed_bytes = sum(p.numel() * 4 for mats in layers for p, _ in mats)
    flags = bl.BL_FLAG_OVERLAP_PREVIOUS
    res = {"packed_GB": packed_bytes / 1e9}
    for B in (1, 16):
        x = synthetic.activations(B, 4096, seed=77, device=dev)
        bufs = {n: torch.empty((B, n), dtype=torch.bfloat16, device=dev) for n in (4096, 11008)}
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
    secondary = None
    if world == 1 and not args.no_secondary:
        import torch
        dev = torch.device("cuda", local_rank)
        flush = _flush_buffer(dev)
        secondary = {"prefill_w1a16": secondary_prefill(dev, peaks, flush),
                     "w1a8_1p3b": secondary_w1a8(dev, peaks, flush)}
        del flush
        secondary["llama7b_linear"] = secondary_llama7b(dev, peaks)
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
        "secondary": secondary,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
