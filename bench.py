#!/usr/bin/env python
"""Benchmark of the NF4 hot path on B200.

One step = the whole path on one weight: quantize (bf16 -> NF4 codes + fp32
absmax), double quantization (E4M3), dequantization (bf16 out), decode GEMV
(batch 1) and prefill GEMM (M = 256), all through the C ABI of libnf4.so.

Workload: the double-quantization case of the reference configs -- a bf16
4096 x 4096 weight ~N(0, 0.02) with 0.1% of entries x20 (seeds 1002/1003) --
with bf16 activations ~N(0, 1) (seeds 1013, 1277).  Inputs rotate over enough
independent copies that every step's working set is cold in the 126 MB L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Beside the step (each timed from its own graph, not part of `value`): the
input gradient dX = dY . Wc (M = 256), the GEMM with an r = 16 adapter, and the
grouped GEMV over the q/k/v projections of an 8B-shaped layer (batch 1).

With N > 1 (torchrun, one process per GPU) every rank runs its own replica
(the path has no cross-GPU exchange); value = all ranks' bytes / max time.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NF4 GEMV/dequant HBM GB/s (% of peak); NF4 GEMM TFLOPS; quantize Gelem/s"
ROWS, COLS, GEMV_B, GEMM_M = 4096, 4096, 1, 256
WORKLOAD = "nf4_path_bf16_4096x4096_outliers_gemv1_gemm256"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNELS = ("quantize", "double_quant", "dequantize", "gemv", "gemm")
NEXT_KERNELS = ("gemm_dx", "gemm_lora", "gemv_grouped")  # timed beside the step, not part of it
QKV_SHAPES = ((4096, 4096), (1024, 4096), (1024, 4096))  # q, k, v of an 8B-shaped layer
LORA_R, LORA_ALPHA = 16, 32.0


def work_per_step(rows=ROWS, cols=COLS, b=GEMV_B, m=GEMM_M):
    """Algorithmic bytes (each operand read once, each output written once at
    its stored width) and flops of every kernel in one step."""
    n = rows * cols
    nb = n // 64
    nb2 = (nb + 255) // 256
    w4 = n // 2 + nb + 4 * nb2 + 4           # NF4 codes + double-quant record
    return {
        "quantize": {"bytes": 2 * n + n // 2 + 4 * nb, "elems": n},
        "double_quant": {"bytes": 4 * nb + nb + 4 * nb2 + 4},
        "dequantize": {"bytes": w4 + 2 * n},
        "gemv": {"bytes": w4 + 2 * b * cols + 2 * b * rows, "flops": 2 * b * n},
        "gemm": {"bytes": w4 + 2 * m * cols + 2 * m * rows, "flops": 2 * m * n},
        "gemm_dx": {"bytes": w4 + 2 * m * rows + 2 * m * cols, "flops": 2 * m * n,
                    "what": f"dX[{m},{cols}] = dY[{m},{rows}] . Wc (input gradient)"},
        "gemv_grouped": {"bytes": sum(r * c // 2 + r * c // 64 + 4 * (r * c // 64 // 256) + 4 + 2 * b * c + 2 * b * r
                                      for r, c in QKV_SHAPES),
                         "flops": sum(2 * b * r * c for r, c in QKV_SHAPES), "bound": "hbm",
                         "what": f"q, k, v of an 8B layer (4096/1024/1024 x 4096) on one x, batch {b}, one launch"},
        "gemm_lora": {"bytes": w4 + 2 * m * cols + 2 * m * rows + 2 * LORA_R * (rows + cols),
                      "flops": 2 * m * n + 2 * m * LORA_R * (rows + cols),
                      "what": f"Y[{m},{rows}] = X . Wc^T + 2 (X . A^T) . B^T, r = {LORA_R} (two launches)"},
    }


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].isdigit():
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = sorted(int(r[1]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": int(rows[0][2]), "samples": len(rows), "reasons": reasons}


# ---------------------------------------------------------------------------- oracle baseline

def oracle_sample_step(sample_rows: int, w_bits, x_bits, X_bits):
    """The same step computed by the CPU oracle on the first `sample_rows` rows
    of the weight (GEMM over all M activation rows).  Returns elapsed seconds
    and the algorithmic bytes of the sample."""
    import oracle
    n = sample_rows * COLS
    t0 = time.perf_counter()
    p, a = oracle.quantize(w_bits[:sample_rows].reshape(-1))
    q, s, mu = oracle.double_quant(a, 256, oracle.DQ_E4M3)
    ah = oracle.absmax_reconstruct(q, s, mu, 256, oracle.DQ_E4M3)
    oracle.dequantize(p, ah, n, 64, "bf16")
    oracle.matmul(p, ah, sample_rows, COLS, x_bits)
    oracle.matmul(p, ah, sample_rows, COLS, X_bits)
    dt = time.perf_counter() - t0
    work = work_per_step(rows=sample_rows)
    return dt, sum(work[k]["bytes"] for k in KERNELS)


def cpu_baseline(sample_rows: int, reps: int = 1):
    import oracle
    from qlora_block_absmax_b200 import synth
    w = synth.bf16_4096x4096_outlier_weight()
    x = synth.activations((GEMV_B, COLS), 1013)
    X = synth.activations((GEMM_M, COLS), 1277)
    oracle.build()
    cores = oracle.get_threads()
    total_t, total_b = 0.0, 0
    for _ in range(reps):
        dt, b = oracle_sample_step(sample_rows, w, x, X)
        total_t += dt
        total_b += b
    return {"value": total_b / total_t / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"whole step on the first {sample_rows} of {ROWS} weight rows "
                      f"(GEMM over all {GEMM_M} activation rows), {reps} rep(s), {total_t:.1f} s",
            "seconds": total_t}


# ---------------------------------------------------------------------------- our arm

def max_over_ranks(v: float, world: int, device) -> float:
    """The largest of the ranks' values (every rank gets it); the value itself with one rank."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(step_bytes: float, steps: int, elapsed_ms_max: float, world: int) -> float:
    """Whole-job GB/s of `world` replicas: every rank's bytes over the slowest rank's device time."""
    return world * step_bytes / (elapsed_ms_max / steps * 1e-3) / 1e9


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import qlora_block_absmax_b200 as nf4
    from qlora_block_absmax_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)

    # ---- inputs (identical values in every copy; distinct memory)
    w_bits = synth.bf16_4096x4096_outlier_weight()
    x_bits = synth.activations((GEMV_B, COLS), 1013)
    X_bits = synth.activations((GEMM_M, COLS), 1277)
    dY_bits = synth.activations((GEMM_M, ROWS), 1279)  # gradient of Y for the input-gradient product
    host_w = torch.from_numpy(w_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    host_x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    host_X = torch.from_numpy(X_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    host_dY = torch.from_numpy(dY_bits.view(np.int16)).view(torch.bfloat16)
    # r = 16, lora_alpha = 32 adapter maps: down ~N(0, 1/cols), up ~N(0, 0.02) (seeds 1281, 1282)
    host_down = torch.from_numpy(synth.f32_to_bf16_bits(
        (synth.rng(1281).standard_normal((LORA_R, COLS)) / np.sqrt(COLS)).astype(np.float32)).view(np.int16)).view(
        torch.bfloat16)
    host_up = torch.from_numpy(synth.f32_to_bf16_bits(
        (synth.rng(1282).standard_normal((ROWS, LORA_R)) * 0.02).astype(np.float32)).view(np.int16)).view(
        torch.bfloat16)
    n = ROWS * COLS
    nb = n // 64
    per_copy = 2 * n + n // 2 + 4 * nb + nb + 2 * n + 2 * GEMM_M * (ROWS + COLS)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = max(4, -(-3 * l2 // per_copy))

    class Copy:
        pass

    # the q, k, v projections of one 8B-shaped layer for the grouped GEMV, drawn on the device (seeds 2000-2002,
    # the whole-model recipe) and quantized by the library at set-up; enough sets (13 MB of codes each) that successive
    # launches read them cold from HBM
    qkv_bytes = sum(r * c * 0.5159 for r, c in QKV_SHAPES)
    qkv_sets = [[nf4.quantize_weight(synth.normal_weights_device(shape, 2000 + j, device=dev))
                 for j, shape in enumerate(QKV_SHAPES)] for _ in range(max(copies, -(-3 * l2 // int(qkv_bytes))))]
    qkv_turn = [0]

    def next_qkv():
        qkv_turn[0] += 1
        return qkv_sets[qkv_turn[0] % len(qkv_sets)]

    cs = []
    for _ in range(copies):
        c = Copy()
        c.w = host_w.to(dev)
        c.x = host_x.to(dev)
        c.X = host_X.to(dev)
        c.packed = torch.empty(n // 2, dtype=torch.uint8, device=dev)
        c.absmax = torch.empty(nb, dtype=torch.float32, device=dev)
        c.q = torch.empty(nb, dtype=torch.uint8, device=dev)
        c.scale = torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev)
        c.mean = torch.empty(1, dtype=torch.float32, device=dev)
        c.ws = torch.zeros(256, dtype=torch.uint8, device=dev)  # double-quant workspace: zeroed once
        c.deq = torch.empty(ROWS, COLS, dtype=torch.bfloat16, device=dev)
        c.y = torch.empty(GEMV_B, ROWS, dtype=torch.bfloat16, device=dev)
        c.Y = torch.empty(GEMM_M, ROWS, dtype=torch.bfloat16, device=dev)
        c.qw = nf4.QuantizedWeight(packed=c.packed, rows=ROWS, cols=COLS, absmax_q=c.q, absmax_scale=c.scale,
                                   absmax_mean=c.mean, dq_code=nf4.NF4_DQ_E4M3)
        c.gws = torch.zeros(max(nf4.gemm_workspace_bytes(c.qw, GEMM_M), 16), dtype=torch.uint8, device=dev)
        c.dY = host_dY.to(dev)
        c.dX = torch.empty(GEMM_M, COLS, dtype=torch.bfloat16, device=dev)
        c.dws = torch.zeros(max(nf4.gemm_dx_workspace_bytes(c.qw, GEMM_M), 16), dtype=torch.uint8, device=dev)
        c.down, c.up = host_down.to(dev), host_up.to(dev)
        c.Yl = torch.empty(GEMM_M, ROWS, dtype=torch.bfloat16, device=dev)
        c.lws = torch.zeros(nf4.gemm_lora_workspace_bytes(c.qw, GEMM_M), dtype=torch.uint8, device=dev)
        c.qkv_y = [torch.empty(GEMV_B, r, dtype=torch.bfloat16, device=dev) for r, _ in QKV_SHAPES]
        cs.append(c)
    stream = torch.cuda.current_stream()

    def calls(c):
        """the five library calls of one step, in order"""
        return (lambda: nf4.quantize(c.w, out=(c.packed, c.absmax)),
                lambda: nf4.double_quant(c.absmax, "e4m3", out=(c.q, c.scale, c.mean), workspace=c.ws),
                lambda: nf4.dequantize(c.qw, torch.bfloat16, out=c.deq),
                lambda: nf4.gemv(c.qw, c.x, out=c.y),
                lambda: nf4.gemm(c.qw, c.X, out=c.Y, workspace=c.gws))

    def next_calls(c):
        """products beyond the step's five calls, timed on their own: the input gradient dX = dY . Wc and the
        GEMM with an r = 16 adapter"""
        return (lambda: nf4.gemm_dx(c.qw, c.dY, out=c.dX, workspace=c.dws),
                lambda: nf4.gemm_lora(c.qw, c.X, c.down, c.up, LORA_ALPHA / LORA_R, out=c.Yl, workspace=c.lws),
                lambda: nf4.gemv_grouped(next_qkv(), c.x, outs=c.qkv_y))

    def step(c):
        for f in calls(c):
            f()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_ms(v: float) -> float:
        return max_over_ranks(v, world, dev)

    for i in range(args.warmup):
        step(cs[i % copies])
    nf4.check_device_error()
    barrier()
    # kernels launched by one step, counted by the library itself
    l0 = nf4.kernel_launches()
    step(cs[0])
    launches_per_step = nf4.kernel_launches() - l0
    # The device-timed region is one CUDA graph holding the K steps (the library
    # launches are chained with programmatic dependent launch), so host-side
    # marshalling cannot gap the GPU timeline.
    def capture(nsteps, only=None, fn=calls):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(nsteps):
                fs = fn(cs[i % copies])
                for f in (fs if only is None else (fs[only],)):
                    f()
        return g

    g_warm = capture(args.warmup)
    g_timed = capture(args.steps)
    # per-kernel times: one graph per library call holding its K launches on the
    # same rotating inputs, timed as a whole (no event nodes between launches)
    g_kernel = [capture(args.steps, j) for j in range(len(KERNELS))]
    g_next = [capture(args.steps, j, next_calls) for j in range(len(NEXT_KERNELS))]
    g_warm.replay()
    for g in g_kernel + g_next:
        g.replay()
    nf4.check_device_error()
    barrier()

    # ---- device-timed region: K steps (one graph replay)
    sampler = ClockSampler(local)
    sampler.start()
    barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    g_timed.replay()
    t_end.record(stream)
    barrier()
    launches = launches_per_step * args.steps
    elapsed_ms = max_ms(t_start.elapsed_time(t_end))
    per_kernel_ms = {}
    for j, k in enumerate(KERNELS):
        k0 = torch.cuda.Event(enable_timing=True)
        k1 = torch.cuda.Event(enable_timing=True)
        k0.record(stream)
        g_kernel[j].replay()
        k1.record(stream)
        barrier()
        per_kernel_ms[k] = max_ms(k0.elapsed_time(k1))
    next_ms = {}
    for j, k in enumerate(NEXT_KERNELS):
        k0 = torch.cuda.Event(enable_timing=True)
        k1 = torch.cuda.Event(enable_timing=True)
        k0.record(stream)
        g_next[j].replay()
        k1.record(stream)
        barrier()
        next_ms[k] = max_ms(k0.elapsed_time(k1))
    clocks = sampler.stop()
    nf4.check_device_error()
    del g_warm, g_timed, g_kernel, g_next

    # ---- end to end through the public API with host buffers
    host_out = {"packed": torch.empty(n // 2, dtype=torch.uint8).pin_memory(),
                "q": torch.empty(nb, dtype=torch.uint8).pin_memory(),
                "scale": torch.empty((nb + 255) // 256, dtype=torch.float32).pin_memory(),
                "mean": torch.empty(1, dtype=torch.float32).pin_memory(),
                "y": torch.empty(GEMV_B, ROWS, dtype=torch.bfloat16).pin_memory(),
                "Y": torch.empty(GEMM_M, ROWS, dtype=torch.bfloat16).pin_memory()}
    h2d = host_w.numel() * 2 + host_x.numel() * 2 + host_X.numel() * 2
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())

    # copies in on one stream, the library calls on the compute stream, results out on a third: the two copy
    # directions and the kernels of neighbouring steps overlap (a step's buffer set is reused only after its
    # results have left)
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    ev_in, ev_out = {}, {}

    def e2e_step(i):
        c = cs[i % copies]
        with torch.cuda.stream(s_in):
            if i - copies in ev_out:
                s_in.wait_event(ev_out[i - copies])
            c.w.copy_(host_w, non_blocking=True)
            c.x.copy_(host_x, non_blocking=True)
            c.X.copy_(host_X, non_blocking=True)
            ev_in[i] = torch.cuda.Event()
            ev_in[i].record(s_in)
        stream.wait_event(ev_in[i])
        step(c)
        done = torch.cuda.Event()
        done.record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done)
            host_out["packed"].copy_(c.packed, non_blocking=True)
            host_out["q"].copy_(c.q, non_blocking=True)
            host_out["scale"].copy_(c.scale, non_blocking=True)
            host_out["mean"].copy_(c.mean, non_blocking=True)
            host_out["y"].copy_(c.y, non_blocking=True)
            host_out["Y"].copy_(c.Y, non_blocking=True)
            ev_out[i] = torch.cuda.Event()
            ev_out[i].record(s_out)

    for i in range(args.warmup):
        e2e_step(i)
    barrier()
    ev_in.clear()
    ev_out.clear()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(args.steps):
        e2e_step(i)
    e1.record(s_out)
    barrier()
    e2e_ms = max_ms(e0.elapsed_time(e1))

    work = work_per_step()
    step_bytes = sum(work[k]["bytes"] for k in KERNELS)
    ms_per_step = elapsed_ms / args.steps
    value = replica_throughput(step_bytes, args.steps, elapsed_ms, world)
    e2e_value = replica_throughput(step_bytes, args.steps, e2e_ms, world)

    peaks, peak_src = load_peaks()
    breakdown = {}
    for k in KERNELS:
        t = per_kernel_ms[k] / args.steps * 1e-3
        d = {"ms": round(t * 1e3, 5), "share": round(per_kernel_ms[k] / sum(per_kernel_ms.values()), 4),
             "gbs": round(work[k]["bytes"] / t / 1e9, 1),
             "frac_hbm": round(work[k]["bytes"] / t / 1e9 / peaks["hbm_gbs"], 4)}
        if "flops" in work[k]:
            d["tflops"] = round(work[k]["flops"] / t / 1e12, 2)
            d["frac_bf16"] = round(work[k]["flops"] / t / 1e12 / peaks["bf16_tflops"], 4)
        if "elems" in work[k]:
            d["gelem_s"] = round(work[k]["elems"] / t / 1e9, 2)
        breakdown[k] = d
    nexts = {}
    for k in NEXT_KERNELS:
        t = next_ms[k] / args.steps * 1e-3
        gbs = work[k]["bytes"] / t / 1e9
        tfl = work[k]["flops"] / t / 1e12
        if work[k].get("bound") == "hbm":
            roof_k = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                      "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": TRAFFIC.get(k)}
        else:
            roof_k = {"bound": "tensor", "achieved": round(tfl, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                      "frac": round(tfl / peaks["bf16_tflops"], 4), "traffic": TRAFFIC.get(k)}
        nexts[k] = {"what": work[k]["what"], "ms": round(t * 1e3, 5), "gbs": round(gbs, 1), "tflops": round(tfl, 2),
                    "roofline": roof_k}
    dom = max(KERNELS, key=lambda k: per_kernel_ms[k])
    t_dom = per_kernel_ms[dom] / args.steps * 1e-3
    if dom == "gemm":
        ach = work[dom]["flops"] / t_dom / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": round(ach, 2), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(ach / peaks["bf16_tflops"], 4)}
    else:
        ach = work[dom]["bytes"] / t_dom / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4)}
    roof["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json burst)" if peak_src == "measured" else "fallback"
    roof["traffic"] = TRAFFIC.get(dom)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "rows": ROWS, "cols": COLS, "gemv_batch": GEMV_B, "gemm_m": GEMM_M,
                   "weight": "bf16 ~N(0,0.02), 0.1% x20 outliers, seeds 1002/1003; NF4 blocksize 64, "
                             "double quant E4M3 blocks of 256",
                   "l2": f"inputs rotate over {copies} copies ({copies * per_copy / 1e6:.0f} MB > L2 "
                         f"{l2 / 1e6:.0f} MB)",
                   "parallelism": "replicas" if world > 1 else "single"},
        "roofline": roof,
        "breakdown": breakdown,
        "next": nexts,
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": int(launches),
        "launch": ("the K timed steps captured in one CUDA graph, launches chained with programmatic dependent "
                   "launch; per-kernel times from one graph of K launches of that kernel; e2e leg launches eagerly, "
                   "copies in, library calls and copies out on three streams overlapping across steps"),
        "clocks": clocks,
        "impl": "ours",
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = {k: (round(v, 4) if isinstance(v, float) else v)
                                for k, v in cpu_baseline(args.cpu_rows, args.cpu_reps).items()}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ncu dram__bytes_read.sum + dram__bytes_write.sum per launch of each kernel at this workload, from the
# --set full capture in profiles/kernels_nf4_path_bf16_4096x4096.md; an entry is removed whenever its kernel
# changes after the capture (the GEMV, the GEMM and the input-gradient GEMM have changed since theirs)
TRAFFIC = {"quantize": 33576192, "double_quant": 1084928, "dequantize": 8679680}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from qlora_block_absmax_b200 import synth
    oracle.build()
    w = synth.bf16_4096x4096_outlier_weight()
    x = synth.activations((GEMV_B, COLS), 1013)
    X = synth.activations((GEMM_M, COLS), 1277)
    rows = args.ref_rows
    for _ in range(args.warmup):
        oracle_sample_step(rows, w, x, X)
    t_total, b_total = 0.0, 0
    for _ in range(args.steps):
        dt, b = oracle_sample_step(rows, w, x, X)
        t_total += dt
        b_total += b
    value = b_total / t_total / 1e9
    cores = oracle.get_threads()
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_total / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "rows": ROWS, "cols": COLS, "gemv_batch": GEMV_B, "gemm_m": GEMM_M},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: whole path on the first {rows} of {ROWS} weight rows "
                                   f"(GEMM over all {GEMM_M} activation rows)"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=ROWS, help="weight rows in the oracle CPU-baseline sample")
    ap.add_argument("--cpu-reps", type=int, default=3, help="repetitions of the oracle CPU-baseline sample")
    ap.add_argument("--ref-rows", type=int, default=1024, help="weight rows per oracle step for --impl reference")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
