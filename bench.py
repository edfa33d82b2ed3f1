"""Benchmark of the 8-bit group-affine quantized linear layer (MlxInt8Weight).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--rows]

Headline workload (one "step"): the decode gemv y = W x over 100 seeded
(weight, x) pairs, N = K = 4096, group_size = 64, m = 1, weights in
u8 group-affine form with BF16 scales/biases, x BF16 N(0,1).  The 100 weights
(1.78 GB) are far larger than the 126 MB L2, so every launch streams its weight
from HBM.  Metric: GEMV HBM GB/s, algorithmic bytes N*K + 4*N*K/gs + 2*K + 2*N
per launch, whole job (all ranks) / device time of the K timed steps.

Under torchrun (N > 1) each rank runs its own 100 pairs (seeds offset by
rank): independent problems, no data-path collective ("scaling": "weak").
Timing: W untimed warm-up steps, then K steps between a barrier +
synchronize on both sides, CUDA events on the launching stream, max over ranks.

Also reported (--rows, on by default at N = 1): dequantize_to on the same 100
weights, the fused decode MLP chain, the small-m gemm shapes and the prefill
gemm on tensor cores at m = 4096 (TFLOP/s), each with its roofline fraction.

--impl reference times the CPU oracle (test infrastructure, single thread) on
a bounded sample of the same workload and prints the same JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

N_PAIRS = 100
D_N, D_K, D_GS = 4096, 4096, 64


def gemv_bytes(N, K, gs, m=1):
    return N * K + 4 * N * K // gs + 2 * K * m + 2 * N * m


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def source_hash(source_files, root=ROOT) -> str:
    """First 16 hex digits of the sha256 over the given files' bytes, in order."""
    import hashlib
    h = hashlib.sha256()
    for f in source_files:
        with open(os.path.join(root, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profile_traffic(kernel_tag: str, source_files, root=ROOT):
    """dram bytes per launch from a committed ncu summary, or None when the
    summary is missing or the kernel sources changed since it was taken."""
    path = os.path.join(root, "profiles", f"{kernel_tag}.md")
    if not os.path.exists(path):
        return None
    digest = source_hash(source_files, root)
    vals = {}
    for line in open(path):
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            v = v.strip()
            if v.startswith("`") and v.count("`") >= 2:
                v = v[1:v.index("`", 1)]  # the first backticked token
            vals[k.strip()] = v
    if vals.get("source_sha256") != digest:
        return None
    try:
        return float(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed regions."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def rank_pair_seeds(rank: int):
    """Seeds of the decode pairs rank `rank` streams: ranks own disjoint,
    consecutive blocks of N_PAIRS problems (weak scaling, no data-path
    collective)."""
    return [rank * N_PAIRS + i for i in range(N_PAIRS)]


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def time_region(fn, steps, warmup, stream, world):
    """W warm-up calls, then `steps` calls between barrier+synchronize; device
    time from CUDA events on `stream`, max over ranks (ms per step)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = e0.elapsed_time(e1) / steps
    return max_over_ranks(ms, world, device="cuda")


def upload_weight(mq, p, s, b, gs, static=True):
    """Load a synthetic weight.  Benchmark weights are loaded once and only
    read, so they carry MLXQ_WEIGHT_STATIC unless static=False."""
    return mq.MlxInt8Weight.load(__import__("synth").weight_blob("w", p, s, b), "w", gs, static=static)


def run_gpu(args):
    import torch
    import synth
    import weight_only_quantized_mlx_b200 as mq

    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    mq.lib()
    peaks = measured_peaks()
    stream = torch.cuda.current_stream()

    # ---- headline: 100 decode gemvs, inputs resident in HBM -----------------
    weights, xs = [], []
    for seed in rank_pair_seeds(rank):
        p, s, b, x = synth.decode_pair(seed, D_N, D_K, D_GS)
        weights.append(upload_weight(mq, p, s, b, D_GS))
        xs.append(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev))
    ys = [torch.empty(D_N, dtype=torch.bfloat16, device=dev) for _ in range(N_PAIRS)]
    s_ptr = stream.cuda_stream
    L = mq.lib()
    import ctypes
    handles = [ctypes.byref(w.handle) for w in weights]
    xp = [x.data_ptr() for x in xs]
    yp = [y.data_ptr() for y in ys]

    def step_on(sp):
        for i in range(N_PAIRS):
            rc = L.mlxq_gemv(handles[i], xp[i], yp[i], sp)
            if rc:
                raise mq.MlxqError(rc, mq.mlxq_last_error())

    # The step's 100 launches are captured once in a CUDA graph and replayed:
    # the launch-bound loop runs without per-launch host overhead.
    step_on(s_ptr)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step_on(torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()

    per_launch = gemv_bytes(D_N, D_K, D_GS)
    rows = {}
    with ClockSampler(dev.index or 0) as clk:
        ms = time_region(graph.replay, args.steps, args.warmup, stream, world)
        ms_eager = time_region(lambda: step_on(s_ptr), args.steps, args.warmup, stream, world)
        # the same graph with the weights' flags cleared: every weight read
        # then waits for the previous launch
        for w in weights:
            w.handle.flags = 0
        step_on(s_ptr)
        torch.cuda.synchronize()
        graph_plain = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_plain):
            step_on(torch.cuda.current_stream().cuda_stream)
        ms_plain = time_region(graph_plain.replay, args.steps, args.warmup, stream, world)
        del graph_plain
        for w in weights:
            w.handle.flags = mq.MLXQ_WEIGHT_STATIC
        # e2e: the public call with host buffers.  Every step copies its 100
        # activation vectors from pinned host memory in one H2D, makes the 100
        # mlxq_gemv calls, and reads the 100 results back in one D2H, all
        # inside the timed region (the copies are batched per step, as a
        # caller holding a step's inputs would do).
        xh = torch.stack([x.cpu() for x in xs]).pin_memory()          # [pairs, K]
        yh = torch.empty(N_PAIRS, D_N, dtype=torch.bfloat16).pin_memory()
        xd = torch.empty(N_PAIRS, D_K, dtype=torch.bfloat16, device=dev)
        yd = torch.empty(N_PAIRS, D_N, dtype=torch.bfloat16, device=dev)

        def step_e2e():
            with torch.cuda.stream(stream):
                xd.copy_(xh, non_blocking=True)
                for i in range(N_PAIRS):
                    mq.mlxq_gemv(weights[i].handle, xd[i], yd[i], stream)
                yh.copy_(yd, non_blocking=True)

        e2e_steps = max(1, args.steps // 4)
        ms_e2e = time_region(step_e2e, e2e_steps, max(3, args.warmup), stream, world)
        if args.rows and world == 1:
            rows = measure_rows(mq, torch, synth, dev, stream, weights, peaks, args)
    mq.mlxq_device_status()
    del graph

    total_bytes = per_launch * N_PAIRS * world
    value = total_bytes / (ms * 1e-3) / 1e9
    e2e_value = total_bytes / (ms_e2e * 1e-3) / 1e9
    achieved = per_launch / (ms * 1e-3 / N_PAIRS) / 1e9
    traffic = profile_traffic("gemv_decode_4096x4096_gs64", [
        "weight_only_quantized_mlx_b200/csrc/gemv_la.cu",
        "weight_only_quantized_mlx_b200/csrc/device_common.cuh"])
    out = {
        "metric": "W8 group-affine GEMV HBM GB/s (% of peak) at m=1; gemm TFLOP/s at m=4096",
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded u8 codes, bf16 scales/biases/activations; no checkpoint)",
        "config": {
            "workload": "decode gemv: 100 seeded (W, x) pairs, N=4096, K=4096, group_size=64, m=1",
            "pairs_per_rank": N_PAIRS,
            "bytes_per_launch": per_launch,
            "l2": "inputs larger than L2 (1.78 GB of weights per rank vs 126 MB L2)",
            "weights": "u8 group-affine, bf16 scale/bias", "activations": "bf16",
            "accumulate": "fp32", "parallelism": f"dp{world} (independent problems)",
            "launch": "CUDA graph of the step's 100 launches",
            "weight_flags": "MLXQ_WEIGHT_STATIC (weights loaded once, never written)",
            "eager_gbs": round(total_bytes / (ms_eager * 1e-3) / 1e9, 1),
            "graph_gbs_without_static_flag": round(total_bytes / (ms_plain * 1e-3) / 1e9, 1),
        },
        "roofline": {
            "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
            "peak_source": peaks["source"], "kernel": "k_gemv_la (mlx_int8_gemv)",
        },
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s",
                "h2d_bytes_per_step": 2 * D_K * N_PAIRS, "d2h_bytes_per_step": 2 * D_N * N_PAIRS},
        "gpu_launches": args.steps * N_PAIRS,
        "clocks": clk.summary(),
    }
    if rows:
        out["rows"] = rows
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_gemv(budget_s=args.cpu_budget)
    for w in weights:
        w.release()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def measure_rows(mq, torch, synth, dev, stream, dec_weights, peaks, args):
    """Secondary rows of the hot path, each timed on its own."""
    torch.manual_seed(20261202)  # every timed input is seeded
    rows = {}
    steps = max(5, args.steps // 10)
    warm = max(3, args.warmup)
    hbm = peaks["hbm_gbs"]

    # dequantize_to over the 100 decode weights; the outputs rotate over 8
    # buffers (268 MB, more than L2) so the writes reach HBM
    outs = [torch.empty(D_N * D_K, dtype=torch.bfloat16, device=dev) for _ in range(8)]

    def deq():
        for i, w in enumerate(dec_weights):
            mq.mlxq_dequant(w.handle, outs[i % len(outs)], stream)
    ms = time_region(deq, steps, warm, stream, 1)
    b = (D_N * D_K + 4 * D_N * D_K // D_GS + 2 * D_N * D_K) * len(dec_weights)
    gbs = b / (ms * 1e-3) / 1e9
    rows["dequant_4096x4096"] = {"value": round(gbs, 1), "unit": "GB/s", "frac_hbm": round(gbs / hbm, 4),
                                 "bytes_per_launch": b // len(dec_weights), "output_buffers": len(outs)}
    del outs

    # quantize: BF16 [4096, 4096] -> codes + tables, 8 sources rotating (268 MB)
    qsrc = [torch.randn(D_N, D_K, device=dev).to(torch.bfloat16) * 0.04 for _ in range(8)]
    qdst = upload_weight(mq, *synth.weight(synth.rng(5000), D_N, D_K, D_GS), D_GS, static=False)
    qturn = [0]

    def quant():
        mq.mlxq_quantize(qsrc[qturn[0] % len(qsrc)], qdst.handle, stream)
        qturn[0] += 1
    ms = time_region(quant, steps, warm, stream, 1)
    b = 2 * D_N * D_K + D_N * D_K + 4 * D_N * D_K // D_GS
    gbs = b / (ms * 1e-3) / 1e9
    rows["quantize_4096x4096"] = {"value": round(gbs, 1), "unit": "GB/s", "frac_hbm": round(gbs / hbm, 4),
                                  "bytes_per_launch": b}
    qdst.release()
    del qsrc

    # a group size the tensor-pipe kernels do not take (8: any-group-size
    # kernels) on the decode shape; 16 weights of 25 MB rotate (400 MB, more
    # than L2)
    gs8 = 8
    w8 = [upload_weight(mq, *synth.weight(synth.rng(7000 + i), D_N, D_K, gs8), gs8) for i in range(16)]
    x8 = torch.randn(D_K, device=dev).to(torch.bfloat16)
    y8 = torch.empty(D_N, dtype=torch.bfloat16, device=dev)
    ms = time_region(lambda: [mq.mlxq_gemv(w.handle, x8, y8, stream) for w in w8], steps, warm, stream, 1)
    b = gemv_bytes(D_N, D_K, gs8) * len(w8)
    gbs = b / (ms * 1e-3) / 1e9
    rows["gemv_4096x4096_gs8"] = {"value": round(gbs, 1), "unit": "GB/s", "frac_hbm": round(gbs / hbm, 4),
                                  "us_per_launch": round(ms * 1e3 / len(w8), 2), "kernel": "k_anygs_gemv"}
    outs = [torch.empty(D_N * D_K, dtype=torch.bfloat16, device=dev) for _ in range(8)]

    def deq8():
        for i, w in enumerate(w8):
            mq.mlxq_dequant(w.handle, outs[i % len(outs)], stream)
    ms = time_region(deq8, steps, warm, stream, 1)
    b = (D_N * D_K + 4 * D_N * D_K // gs8 + 2 * D_N * D_K) * len(w8)
    gbs = b / (ms * 1e-3) / 1e9
    rows["dequant_4096x4096_gs8"] = {"value": round(gbs, 1), "unit": "GB/s", "frac_hbm": round(gbs / hbm, 4),
                                     "kernel": "k_dequant_anygs"}
    del outs
    for w in w8:
        w.release()

    # fused decode MLP: gate, up (14336x4096) then silu_gate_resid down (4096x14336)
    D, F, gs = 4096, 14336, 64
    mlps = []
    for j in range(4):  # 4 layers' weights (750 MB) rotate so L2 cannot hold them
        g = synth.rng(1000 + j)
        ws = [upload_weight(mq, *synth.weight(g, F, D, gs), gs), upload_weight(mq, *synth.weight(g, F, D, gs), gs),
              upload_weight(mq, *synth.weight(g, D, F, gs), gs)]
        mlps.append(ws)
    g = synth.rng(2000)
    x = torch.from_numpy(synth.activations(g, D).view(np.int16)).view(torch.bfloat16).to(dev)
    xr = torch.from_numpy(synth.activations(g, D).view(np.int16)).view(torch.bfloat16).to(dev)
    gate = torch.empty(F, dtype=torch.bfloat16, device=dev)
    up = torch.empty(F, dtype=torch.bfloat16, device=dev)
    y = torch.empty(D, dtype=torch.bfloat16, device=dev)

    def mlp():
        for wg, wu, wd in mlps:
            mq.mlxq_gemv(wg.handle, x, gate, stream)
            mq.mlxq_gemv(wu.handle, x, up, stream)
            mq.mlxq_gemv_silu_gate_resid(wd.handle, gate, up, xr, y, stream)
    ms = time_region(mlp, steps, warm, stream, 1)
    b = 2 * gemv_bytes(F, D, gs) + (D * F + 4 * D * F // gs + 4 * F + 4 * D)
    us = ms * 1e3 / len(mlps)
    gbs = b / (us * 1e-6) / 1e9
    rows["fused_mlp_decode"] = {"value": round(gbs, 1), "unit": "GB/s", "us_per_mlp": round(us, 2),
                                "frac_hbm": round(gbs / hbm, 4), "bytes_per_mlp": b}
    for ws in mlps:
        for w in ws:
            w.release()

    # the same MLP with gate and up loaded as one [2F, D] weight: two launches
    # per layer (gemv into [gate | up], then silu_gate_resid)
    mlps = []
    for j in range(4):
        g = synth.rng(1000 + j)
        pg, sg, bg = synth.weight(g, F, D, gs)
        pu, su, bu = synth.weight(g, F, D, gs)
        wgu = upload_weight(mq, np.concatenate([pg, pu]), np.concatenate([sg, su]), np.concatenate([bg, bu]), gs)
        mlps.append((wgu, upload_weight(mq, *synth.weight(g, D, F, gs), gs)))
    gu = torch.empty(2 * F, dtype=torch.bfloat16, device=dev)

    def mlp2():
        for wgu, wd in mlps:
            mq.mlxq_gemv(wgu.handle, x, gu, stream)
            mq.mlxq_gemv_silu_gate_resid(wd.handle, gu[:F], gu[F:], xr, y, stream)
    ms = time_region(mlp2, steps, warm, stream, 1)
    us = ms * 1e3 / len(mlps)
    gbs = b / (us * 1e-6) / 1e9
    rows["fused_mlp_decode_concat"] = {"value": round(gbs, 1), "unit": "GB/s", "us_per_mlp": round(us, 2),
                                       "frac_hbm": round(gbs / hbm, 4), "bytes_per_mlp": b, "launches_per_mlp": 2}
    for ws in mlps:
        for w in ws:
            w.release()

    # small-m batched decode: (N, K) in {(28672, 8192), (8192, 28672)},
    # group_size in {32, 64, 128} (each weight 235 MB, more than L2)
    for gs_m in (64, 32, 128):
        for (N, K) in ((28672, 8192), (8192, 28672)):
            w = upload_weight(mq, *synth.weight(synth.rng(3000 + N + gs_m), N, K, gs_m), gs_m)
            for m in (1, 2, 4, 8, 16, 32):
                X = torch.randn(m, K, device=dev).to(torch.bfloat16)
                Y = torch.empty(m, N, dtype=torch.bfloat16, device=dev)
                ms = time_region(lambda: mq.mlxq_gemm(w.handle, X, Y, m, stream), steps, warm, stream, 1)
                b = gemv_bytes(N, K, gs_m, m)
                tag = f"smallm_{N}x{K}_m{m}" + ("" if gs_m == 64 else f"_gs{gs_m}")
                rows[tag] = {"value": round(b / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                             "tflops": round(2 * m * N * K / (ms * 1e-3) / 1e12, 2),
                             "frac_hbm": round(b / (ms * 1e-3) / 1e9 / hbm, 4),
                             "us": round(ms * 1e3, 2)}
            w.release()

    # prefill gemm (tensor cores), m in {512, 2048, 4096, 8192}: m >= 2048
    # fills every SM with whole tiles; at m = 512 there are fewer tiles than
    # SMs, so each tile's K is split (three weight copies, 183 MB, taken in
    # turn: larger than L2)
    for (N, K) in ((4096, 14336), (14336, 4096)):
        ws = [upload_weight(mq, *synth.weight(synth.rng(4000 + N + i), N, K, 64), 64) for i in range(3)]
        for m in (512, 2048, 4096, 8192):
            X = torch.randn(m, K, device=dev).to(torch.bfloat16)
            Y = torch.empty(m, N, dtype=torch.bfloat16, device=dev)
            turn = [0]

            def call():
                w = ws[turn[0] % len(ws)]
                turn[0] += 1
                mq.mlxq_gemm_with(w.handle, X, Y, m, mq.MLXQ_GEMM_TCGEN05, stream)
            try:
                ms = time_region(call, steps, warm, stream, 1)
                tf = 2 * m * N * K / (ms * 1e-3) / 1e12
                rows[f"prefill_{N}x{K}_m{m}"] = {"value": round(tf, 1), "unit": "TFLOP/s",
                                                 "frac_bf16": round(tf / peaks["bf16_tflops"], 4),
                                                 "ms": round(ms, 4)}
            except mq.MlxqError as e:
                rows[f"prefill_{N}x{K}_m{m}"] = {"value": None, "unit": "TFLOP/s", "unavailable": str(e)}
        for w in ws:
            w.release()
    return rows


# ---------------------------------------------------------------------------
# CPU oracle (baseline / reference arm)
# ---------------------------------------------------------------------------
def cpu_baseline_gemv(budget_s: float = 12.0):
    """The oracle's gemv, single-threaded, on as many of the decode pairs as
    fit in about `budget_s` seconds; GB/s over the same algorithmic bytes."""
    import oracle
    import synth
    done, t_total = 0, 0.0
    for i in range(N_PAIRS):
        p, s, b, x = synth.decode_pair(i, D_N, D_K, D_GS)
        t0 = time.perf_counter()
        oracle.gemv(p, s, b, D_GS, x)
        t_total += time.perf_counter() - t0
        done += 1
        if t_total > budget_s:
            break
    gbs = gemv_bytes(D_N, D_K, D_GS) * done / t_total / 1e9
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{done} of the {N_PAIRS} decode pairs (N=K=4096, gs=64), one oracle gemv each",
            "host_cpus": os.cpu_count(), "cpu_model": cpu_model()}


def cpu_model() -> str:
    """The host CPU's model name (first 'model name' line of /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return  # other ranks exit without work
    import oracle
    import synth
    per_step_pairs = 2  # bounded sample per step (about 0.2 s of CPU per step)
    for i in range(args.warmup):
        p, s, b, x = synth.decode_pair(i, D_N, D_K, D_GS)
        oracle.gemv(p, s, b, D_GS, x)
    data = [synth.decode_pair(i, D_N, D_K, D_GS) for i in range(per_step_pairs)]
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for (p, s, b, x) in data:
            oracle.gemv(p, s, b, D_GS, x)
    dt = time.perf_counter() - t0
    ms = dt * 1e3 / args.steps
    gbs = gemv_bytes(D_N, D_K, D_GS) * per_step_pairs / (ms * 1e-3) / 1e9
    sample = f"{per_step_pairs} decode pairs per step (N=K=4096, gs=64), single-threaded oracle gemv"
    out = {
        "metric": "W8 group-affine GEMV HBM GB/s (% of peak) at m=1; gemm TFLOP/s at m=4096",
        "value": round(gbs, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "decode gemv: 100 seeded (W, x) pairs, N=4096, K=4096, group_size=64, m=1",
                   "sample_pairs_per_step": per_step_pairs},
        "impl": "reference",
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample,
                         "host_cpus": os.cpu_count(), "cpu_model": cpu_model()},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def run_case(args):
    """--case KIND:N:K:GS[:M]: run one kernel `--steps` times on a seeded
    weight, no timing line (the command the committed ncu summaries use).
    KIND is dequant, quantize, gemv, silu, resid, gemm (auto), smallm, rows or tc."""
    import torch
    import synth
    import weight_only_quantized_mlx_b200 as mq
    parts = args.case.split(":")
    kind, N, K, gs = parts[0], int(parts[1]), int(parts[2]), int(parts[3])
    m = int(parts[4]) if len(parts) > 4 else 1
    torch.cuda.set_device(0)
    g = synth.rng(7)
    w = upload_weight(mq, *synth.weight(g, N, K, gs), gs)
    dev = torch.device("cuda", 0)
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    X = to_dev(synth.activations(g, m, K))
    gate, up = to_dev(synth.activations(g, K)), to_dev(synth.activations(g, K))
    r = to_dev(synth.activations(g, N))
    Y = torch.empty(m, N, dtype=torch.bfloat16, device=dev)
    out = torch.empty(N * K, dtype=torch.bfloat16, device=dev) if kind == "dequant" else None
    wsrc = to_dev(synth.activations(g, N, K)) if kind == "quantize" else None
    if kind == "quantize":
        w.release()
        w = upload_weight(mq, *synth.weight(g, N, K, gs), gs, static=False)  # the destination is written
    kernel = {"gemm": mq.MLXQ_GEMM_AUTO, "smallm": mq.MLXQ_GEMM_SMALLM, "rows": mq.MLXQ_GEMM_ROWS,
              "tc": mq.MLXQ_GEMM_TCGEN05}.get(kind)
    for _ in range(args.steps):
        if kind == "dequant":
            mq.mlxq_dequant(w.handle, out)
        elif kind == "quantize":
            mq.mlxq_quantize(wsrc, w.handle)
        elif kind == "gemv":
            mq.mlxq_gemv(w.handle, X, Y)
        elif kind == "silu":
            mq.mlxq_gemv_silu_gate(w.handle, gate, up, Y)
        elif kind == "resid":
            mq.mlxq_gemv_silu_gate_resid(w.handle, gate, up, r, Y)
        else:
            mq.mlxq_gemm_with(w.handle, X, Y, m, kernel)
    torch.cuda.synchronize()
    mq.mlxq_device_status()
    w.release()
    print(f"case {args.case}: {args.steps} launches ok")


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="mlxq", choices=["mlxq", "reference"])
    ap.add_argument("--rows", dest="rows", action="store_true", default=True)
    ap.add_argument("--no-rows", dest="rows", action="store_false")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--case", default=None, help="KIND:N:K:GS[:M] single-kernel run for profiling")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # at least 3 warm-up steps, always
    if args.case:
        run_case(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
