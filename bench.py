#!/usr/bin/env python
"""Benchmark of the NF4 hot path on B200.

One step = the whole path on one weight: quantize (bf16 -> NF4 codes + fp32
absmax), double quantization (E4M3), dequantization (bf16 out), decode GEMV
(batch 1) and prefill GEMM (M = 256), all through the C ABI of libnf4.so.

Workload of the step: the double-quantization case of the reference configs --
a bf16 4096 x 4096 weight ~N(0, 0.02) with 0.1% of entries x20 (seeds
1002/1003) -- with bf16 activations ~N(0, 1) (seeds 1013, 1277).  Inputs rotate
over enough independent copies that every step's working set is cold in the
126 MB L2.

Beside the step, `configs` reports every workload of the reference configs, each
leg timed from its own CUDA graph of K to 64 launches (about 2 ms of work) over inputs rotating through at
least 3x the L2 (or larger than it), with its own roofline fraction:
  1  fp32 1024x1024 quantize and dequantize (fp32 out), no double quant
  2  bf16 4096x4096 quantize, double quant E4M3 and INT8
  3  decode GEMV at 4096x4096, 14336x4096, 4096x14336, batch 1/4/8
  4  GEMM 14336x4096 at M = 16, 64, 256, 1024, 4096
  5  the 8B-shaped model (224 weights): quantize + double quant of every weight,
     and one decode GEMV pass over all of them (one launch) at batch 1/4/8
and `next` the input gradient, the adapter GEMM and the grouped q/k/v GEMV.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--quick]

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
GEMV_SHAPES = ((4096, 4096), (14336, 4096), (4096, 14336))
GEMV_BATCHES = (1, 4, 8)
GEMM_SHAPE = (14336, 4096)
GEMM_MS = (16, 64, 256, 1024, 4096)
LORA_R, LORA_ALPHA = 16, 32.0


def record_bytes(rows, cols, dq=True):
    """Stored bytes of a quantized [rows, cols] weight: codes + scales (double-quant record, or fp32 absmax)."""
    n = rows * cols
    nb = -(-n // 64)
    return -(-n // 2) + (nb + 4 * -(-nb // 256) + 4 if dq else 4 * nb)


def gemv_work(rows, cols, b):
    return {"bytes": record_bytes(rows, cols) + 2 * b * cols + 2 * b * rows, "flops": 2 * b * rows * cols}


def gemm_work(rows, cols, m):
    return {"bytes": record_bytes(rows, cols) + 2 * m * cols + 2 * m * rows, "flops": 2 * m * rows * cols}


def work_per_step(rows=ROWS, cols=COLS, b=GEMV_B, m=GEMM_M):
    """Algorithmic bytes (each operand read once, each output written once at its stored width) and flops of every
    kernel in one step."""
    n = rows * cols
    nb = n // 64
    nb2 = (nb + 255) // 256
    w4 = record_bytes(rows, cols)
    return {
        "quantize": {"bytes": 2 * n + n // 2 + 4 * nb, "elems": n},
        "double_quant": {"bytes": 4 * nb + nb + 4 * nb2 + 4},
        "dequantize": {"bytes": w4 + 2 * n},
        "gemv": gemv_work(rows, cols, b),
        "gemm": gemm_work(rows, cols, m),
        "gemm_dx": {"bytes": w4 + 2 * m * rows + 2 * m * cols, "flops": 2 * m * n,
                    "what": f"dX[{m},{cols}] = dY[{m},{rows}] . Wc (input gradient)"},
        "gemv_grouped": {"bytes": sum(gemv_work(r, c, b)["bytes"] for r, c in QKV_SHAPES),
                         "flops": sum(2 * b * r * c for r, c in QKV_SHAPES), "bound": "hbm",
                         "what": f"q, k, v of an 8B layer (4096/1024/1024 x 4096) on one x, batch {b}, one launch"},
        "gemm_lora": {"bytes": w4 + 2 * m * cols + 2 * m * rows + 2 * LORA_R * (rows + cols),
                      "flops": 2 * m * n + 2 * m * LORA_R * (rows + cols),
                      "what": f"Y[{m},{rows}] = X . Wc^T + 2 (X . A^T) . B^T, r = {LORA_R} (two launches)"},
    }


def model_shapes():
    from qlora_block_absmax_b200 import synth
    return [(layer, p, rows, cols) for layer in range(synth.LLAMA8B_LAYERS)
            for p, (_, rows, cols) in enumerate(synth.LLAMA8B_LAYER)]


def model_work(b):
    """the 8B-shaped stack: quantize + double quant of every weight from bf16, and one GEMV pass at batch b"""
    shapes = model_shapes()
    # quantize: bf16 in, codes + fp32 absmax out; double quant: absmax in, 8-bit codes + scales + mean out
    quant = sum(2 * r * c + r * c // 2 + 4 * (r * c // 64) for _, _, r, c in shapes)
    dq = sum(4 * (r * c // 64) + (record_bytes(r, c) - r * c // 2) for _, _, r, c in shapes)
    return {"quantize_pass": {"bytes": quant + dq, "elems": sum(r * c for _, _, r, c in shapes)},
            "gemv_pass": {"bytes": sum(gemv_work(r, c, b)["bytes"] for _, _, r, c in shapes),
                          "flops": sum(2 * b * r * c for _, _, r, c in shapes)}}


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
    """The oracle on a bounded sample of the step, on all host cores and on one."""
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
    oracle.set_threads(1)
    one_rows = max(16, sample_rows // 16)
    t1, b1 = oracle_sample_step(one_rows, w, x, X)
    oracle.set_threads(cores)
    return {"value": total_b / total_t / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"whole step on the first {sample_rows} of {ROWS} weight rows "
                      f"(GEMM over all {GEMM_M} activation rows), {reps} rep(s), {total_t:.1f} s",
            "seconds": total_t, "single_core_value": b1 / t1 / 1e9,
            "single_core_sample": f"whole step on the first {one_rows} weight rows, 1 thread, {t1:.1f} s",
            "cpu_model": cpu_model()}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


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


def copies_for(per_set_bytes: int, l2: int, least: int = 2) -> int:
    """Input sets to rotate so that consecutive launches read cold data: at least 3x the L2 in total."""
    return max(least, -(-3 * l2 // max(1, per_set_bytes)))


def roofline_entry(work: dict, seconds: float, peaks: dict, bound: str) -> dict:
    """achieved, peak and fraction of one leg: bytes against the HBM copy peak, or flops against the bf16 burst peak"""
    if bound == "tensor":
        ach = work["flops"] / seconds / 1e12
        return {"bound": "tensor", "achieved": round(ach, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(ach / peaks["bf16_tflops"], 4)}
    ach = work["bytes"] / seconds / 1e9
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(ach / peaks["hbm_gbs"], 4)}


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
    stream = torch.cuda.current_stream()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    peaks, peak_src = load_peaks()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_ms(v: float) -> float:
        return max_over_ranks(v, world, dev)

    def bf16_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    def graph_of(calls, n):
        """one CUDA graph of n launches, launch i = calls[i % len(calls)] (each on its own input set)"""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                calls[i % len(calls)]()
        return g

    def time_calls(calls, n=None, launches_per_call=1):
        """device ms per call: a warm replay, then a timed replay of a graph of n calls rotating over the sets.
        Short calls get up to 64 per graph (the graph launch's own fixed cost then is a small part of each call's
        share) while a graph stays near 2 ms of work, so a long call is still timed as a burst."""
        for c in calls[:3]:
            c()
        if n is None:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            calls[3 % len(calls)]()
            e1.record(stream)
            torch.cuda.synchronize()
            n = max(args.steps, min(64, int(2.0 / max(e0.elapsed_time(e1), 1e-3))))
        g = graph_of(calls, n)
        g.replay()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        barrier()
        del g
        return max_ms(e0.elapsed_time(e1)) / n

    # ------------------------------------------------------------------ the step (config 2 weight)
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
    copies = copies_for(per_copy, l2, 4)

    class Copy:
        pass

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
        cs.append(c)

    def calls(c):
        """the five library calls of one step, in order"""
        return (lambda: nf4.quantize(c.w, out=(c.packed, c.absmax)),
                lambda: nf4.double_quant(c.absmax, "e4m3", out=(c.q, c.scale, c.mean), workspace=c.ws),
                lambda: nf4.dequantize(c.qw, torch.bfloat16, out=c.deq),
                lambda: nf4.gemv(c.qw, c.x, out=c.y),
                lambda: nf4.gemm(c.qw, c.X, out=c.Y, workspace=c.gws))

    def step(c):
        for f in calls(c):
            f()

    for i in range(args.warmup):
        step(cs[i % copies])
    nf4.check_device_error()
    barrier()
    l0 = nf4.kernel_launches()  # kernels launched by one step, counted by the library itself
    step(cs[0])
    launches_per_step = nf4.kernel_launches() - l0

    # The device-timed region is one CUDA graph holding the K steps (the library launches are chained with
    # programmatic dependent launch), so host-side marshalling cannot gap the GPU timeline.
    def capture(nsteps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(nsteps):
                step(cs[i % copies])
        return g

    g_warm = capture(args.warmup)
    g_timed = capture(args.steps)
    g_warm.replay()
    nf4.check_device_error()
    barrier()

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
    del g_warm, g_timed

    # Per-kernel times of the step: one graph per library call holding K launches, each leg over its own input sets
    # (>= 3x L2 of what that call reads): copies of the step's source weight for quantize, of its absmax values for
    # double quant, and of its quantized record (codes, 8-bit scale codes, scales, mean) for the products.
    c0 = cs[0]
    per_kernel_ms = {}
    k_q = copies_for(2 * n + n // 2 + 4 * nb, l2)
    qsets = [(cs[i].w if i < copies else c0.w.clone(), torch.empty_like(c0.packed), torch.empty_like(c0.absmax))
             for i in range(k_q)]
    per_kernel_ms["quantize"] = time_calls([lambda s=s: nf4.quantize(s[0], out=(s[1], s[2])) for s in qsets])
    del qsets
    k_dq = copies_for(5 * nb, l2)
    dqsets = [(c0.absmax.clone(), torch.empty_like(c0.q), torch.empty_like(c0.scale), torch.empty_like(c0.mean),
               torch.zeros(256, dtype=torch.uint8, device=dev)) for _ in range(k_dq)]
    dq_calls = [lambda s=s: nf4.double_quant(s[0], "e4m3", out=s[1:4], workspace=s[4]) for s in dqsets]
    per_kernel_ms["double_quant"] = time_calls(dq_calls)
    k_rec = copies_for(record_bytes(ROWS, COLS), l2)
    recs = [nf4.QuantizedWeight(packed=c0.packed.clone(), rows=ROWS, cols=COLS, absmax_q=c0.q.clone(),
                                absmax_scale=c0.scale.clone(), absmax_mean=c0.mean.clone(), dq_code=nf4.NF4_DQ_E4M3)
            for _ in range(k_rec)]
    # a fresh output per call as well (every write goes to lines not in L2, like every read)
    deq_out = [torch.empty(ROWS, COLS, dtype=torch.bfloat16, device=dev) for _ in range(k_rec)]
    per_kernel_ms["dequantize"] = time_calls([lambda q=q, o=o: nf4.dequantize(q, torch.bfloat16, out=o)
                                              for q, o in zip(recs, deq_out)])
    del deq_out
    ys = [torch.empty(GEMV_B, ROWS, dtype=torch.bfloat16, device=dev) for _ in range(k_rec)]
    per_kernel_ms["gemv"] = time_calls([lambda q=q, y=y: nf4.gemv(q, c0.x, out=y) for q, y in zip(recs, ys)])
    Xs = [cs[i % copies].X for i in range(3)]
    Ys = [torch.empty(GEMM_M, ROWS, dtype=torch.bfloat16, device=dev) for _ in range(k_rec)]
    per_kernel_ms["gemm"] = time_calls([lambda q=q, X=Xs[i % 3], Y=Ys[i]: nf4.gemm(q, X, out=Y, workspace=c0.gws)
                                        for i, q in enumerate(recs)])
    dYs = [cs[i % copies].dY for i in range(3)]
    dXs = [torch.empty(GEMM_M, COLS, dtype=torch.bfloat16, device=dev) for _ in range(k_rec)]
    next_ms = {
        "gemm_dx": time_calls([lambda q=q, dY=dYs[i % 3], dX=dXs[i]: nf4.gemm_dx(q, dY, out=dX, workspace=c0.dws)
                               for i, q in enumerate(recs)]),
        "gemm_lora": time_calls([lambda q=q, X=Xs[i % 3], Y=Ys[i]: nf4.gemm_lora(q, X, c0.down, c0.up,
                                                                               LORA_ALPHA / LORA_R, out=Y,
                                                                               workspace=c0.lws)
                                 for i, q in enumerate(recs)]),
    }
    del recs, ys, Ys, dXs

    # ------------------------------------------------------------------ configs
    configs = {}
    cfg_launches = 0

    def quantized_set(shape, count, seed0):
        return [nf4.quantize_weight(synth.normal_weights_device(shape, seed0 + i, device=dev)) for i in range(count)]

    # config 1: fp32 1024 x 1024 ~N(0, 0.02), quantize + dequantize (fp32 out), no double quant
    w1 = torch.from_numpy(synth.fp32_1024x1024_weight()).to(dev)
    n1 = w1.numel()
    c1_work_q = {"bytes": 4 * n1 + n1 // 2 + 4 * (n1 // 64), "elems": n1}
    c1_work_d = {"bytes": n1 // 2 + 4 * (n1 // 64) + 4 * n1, "elems": n1}
    k1 = copies_for(c1_work_q["bytes"], l2)
    sets1 = []
    for _ in range(k1):
        src = w1.clone()
        p_ = torch.empty(n1 // 2, dtype=torch.uint8, device=dev)
        a_ = torch.empty(n1 // 64, dtype=torch.float32, device=dev)
        o_ = torch.empty(1024, 1024, dtype=torch.float32, device=dev)
        sets1.append((src, p_, a_, o_, nf4.QuantizedWeight(packed=p_, rows=1024, cols=1024, absmax=a_)))
    tq = time_calls([lambda s=s: nf4.quantize(s[0], out=(s[1], s[2])) for s in sets1]) * 1e-3
    td = time_calls([lambda s=s: nf4.dequantize(s[4], torch.float32, out=s[3]) for s in sets1]) * 1e-3
    cfg_launches += 2 * args.steps
    configs["1_fp32_1024x1024"] = {
        "what": "fp32 1024x1024 ~N(0,0.02) seed 1001, blocksize 64, no double quant; quantize, then dequantize to "
                f"fp32; each leg a graph of {args.steps} launches over {k1} input sets",
        "quantize": {"us": round(tq * 1e6, 3), "gelem_s": round(n1 / tq / 1e9, 2),
                     "roofline": roofline_entry(c1_work_q, tq, peaks, "hbm")},
        "dequantize_f32": {"us": round(td * 1e6, 3), "gelem_s": round(n1 / td / 1e9, 2),
                           "roofline": roofline_entry(c1_work_d, td, peaks, "hbm")}}
    del sets1, w1

    # config 2: the step's weight; its quantize and E4M3 double quant are the step's legs, plus INT8 double quant
    t_int8 = time_calls([lambda s=s: nf4.double_quant(s[0], "int8", out=s[1:4], workspace=s[4]) for s in dqsets]) * 1e-3
    t_e4m3 = per_kernel_ms["double_quant"] * 1e-3
    del dqsets
    cfg_launches += args.steps
    work = work_per_step()
    tq2 = per_kernel_ms["quantize"] * 1e-3
    configs["2_bf16_4096x4096_dq"] = {
        "what": "bf16 4096x4096 ~N(0,0.02), 0.1% x20 outliers (seeds 1002/1003); quantize, then double quant of the "
                f"262144 absmax values in blocks of 256 (quantize over {k_q} source copies, double quant over "
                f"{k_dq} absmax copies)",
        "quantize": {"us": round(tq2 * 1e6, 3), "gelem_s": round(n / tq2 / 1e9, 2),
                     "roofline": roofline_entry(work["quantize"], tq2, peaks, "hbm")},
        "double_quant_e4m3": {"us": round(t_e4m3 * 1e6, 3),
                              "roofline": roofline_entry(work["double_quant"], t_e4m3, peaks, "hbm")},
        "double_quant_int8": {"us": round(t_int8 * 1e6, 3),
                              "roofline": roofline_entry(work["double_quant"], t_int8, peaks, "hbm")}}

    # config 3: decode GEMV, cold weights (seeds 1010-1012 + copy), x seed 1013
    cfg3 = {}
    for si, (r, c) in enumerate(GEMV_SHAPES):
        k3 = copies_for(record_bytes(r, c), l2)
        ws = quantized_set((r, c), k3, 1010 + si * 100)
        for b in GEMV_BATCHES:
            x = synth.activations_device((b, c), 1013, device=dev)
            ys = [torch.empty(b, r, dtype=torch.bfloat16, device=dev) for _ in range(k3)]
            t = time_calls([lambda q=q, y=y, x=x: nf4.gemv(q, x, out=y) for q, y in zip(ws, ys)]) * 1e-3
            cfg_launches += args.steps
            cfg3[f"{r}x{c}_b{b}"] = {"us": round(t * 1e6, 3),
                                     "roofline": roofline_entry(gemv_work(r, c, b), t, peaks, "hbm")}
        del ws
    configs["3_gemv"] = dict(
        what=f"decode GEMV y = x . Wc^T, NF4 + E4M3 double quant, weights ~N(0,0.02) from the device generator, "
             f"x ~N(0,1) bf16 (seed 1013); each leg rotates over weight copies of >= 3x the L2 in total", **cfg3)

    # config 4: GEMM 14336 x 4096 at M = 16 ... 4096 (M <= 64: HBM roofline; M >= 256: tensor roofline)
    r4, c4 = GEMM_SHAPE
    k4w = copies_for(record_bytes(r4, c4), l2)
    ws4 = quantized_set((r4, c4), k4w, 1020)
    cfg4 = {}
    for m in GEMM_MS:
        per = record_bytes(r4, c4) + 2 * m * (r4 + c4)
        k4 = min(k4w, copies_for(per, l2))
        Xs = [synth.activations_device((m, c4), 1021 + m + i, device=dev) for i in range(min(k4, 3))]
        Ys = [torch.empty(m, r4, dtype=torch.bfloat16, device=dev) for _ in range(k4)]
        wsp = torch.zeros(max(16, nf4.gemm_workspace_bytes(ws4[0], m)), dtype=torch.uint8, device=dev)
        t = time_calls([lambda q=ws4[i], X=Xs[i % len(Xs)], Y=Ys[i], wsp=wsp: nf4.gemm(q, X, out=Y, workspace=wsp)
                        for i in range(k4)]) * 1e-3
        cfg_launches += args.steps
        wk = gemm_work(r4, c4, m)
        bound = "tensor" if m >= 256 else "hbm"
        cfg4[f"M{m}"] = {"us": round(t * 1e6, 3), "tflops": round(wk["flops"] / t / 1e12, 2),
                         "gbs": round(wk["bytes"] / t / 1e9, 1), "roofline": roofline_entry(wk, t, peaks, bound)}
        del Xs, Ys
    del ws4
    configs["4_gemm_14336x4096"] = dict(
        what="prefill GEMM Y = X . Wc^T, W 14336x4096 NF4 + E4M3 double quant (seed 1020), X ~N(0,1) bf16 "
             "(seed 1021 + M); tcgen05 kernel for M > 64, the GEMV kernels for M <= 64", **cfg4)

    # config 5: the 8B-shaped model (32 layers x q,k,v,o,gate,up,down) ~N(0, 0.02), seeds 2000 + 7 layer + proj
    if not args.quick:
        configs["5_model_8b"] = model_config(args, nf4, synth, dev, time_calls, peaks)
        cfg_launches += configs["5_model_8b"].pop("_launches")

    # the grouped q/k/v GEMV beside the step (seeds 2000-2002, enough sets that every launch reads cold codes)
    qkv_bytes = sum(record_bytes(r, c) for r, c in QKV_SHAPES)
    qkv_sets = [[nf4.quantize_weight(synth.normal_weights_device(shape, 2000 + j, device=dev))
                 for j, shape in enumerate(QKV_SHAPES)] for _ in range(copies_for(qkv_bytes, l2))]
    qkv_y = [torch.empty(GEMV_B, r, dtype=torch.bfloat16, device=dev) for r, _ in QKV_SHAPES]
    next_ms["gemv_grouped"] = time_calls([lambda s=s: nf4.gemv_grouped(s, cs[0].x, outs=qkv_y) for s in qkv_sets])
    del qkv_sets
    clocks = sampler.stop()
    nf4.check_device_error()

    # ---- end to end through the public API with host buffers
    host_out = {"packed": torch.empty(n // 2, dtype=torch.uint8).pin_memory(),
                "q": torch.empty(nb, dtype=torch.uint8).pin_memory(),
                "scale": torch.empty((nb + 255) // 256, dtype=torch.float32).pin_memory(),
                "mean": torch.empty(1, dtype=torch.float32).pin_memory(),
                "deq": torch.empty(ROWS, COLS, dtype=torch.bfloat16).pin_memory(),
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
            host_out["deq"].copy_(c.deq, non_blocking=True)
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

    step_bytes = sum(work[k]["bytes"] for k in KERNELS)
    ms_per_step = elapsed_ms / args.steps
    value = replica_throughput(step_bytes, args.steps, elapsed_ms, world)
    e2e_value = replica_throughput(step_bytes, args.steps, e2e_ms, world)

    breakdown = {}
    for k in KERNELS:
        t = per_kernel_ms[k] * 1e-3
        d = {"ms": round(t * 1e3, 5), "share": round(per_kernel_ms[k] / sum(per_kernel_ms.values()), 4),
             "gbs": round(work[k]["bytes"] / t / 1e9, 1),
             "frac_hbm": round(work[k]["bytes"] / t / 1e9 / peaks["hbm_gbs"], 4)}
        if "flops" in work[k]:
            d["tflops"] = round(work[k]["flops"] / t / 1e12, 2)
            d["frac_bf16"] = round(work[k]["flops"] / t / 1e12 / peaks["bf16_tflops"], 4)
        if "elems" in work[k]:
            d["gelem_s"] = round(work[k]["elems"] / t / 1e9, 2)
        d["traffic"] = TRAFFIC.get(k)  # ncu DRAM bytes per launch (cold), or None
        breakdown[k] = d
    nexts = {}
    for k in NEXT_KERNELS:
        t = next_ms[k] * 1e-3
        roof_k = roofline_entry(work[k], t, peaks, "hbm" if work[k].get("bound") == "hbm" else "tensor")
        roof_k["traffic"] = TRAFFIC.get(k)
        nexts[k] = {"what": work[k]["what"], "ms": round(t * 1e3, 5), "gbs": round(work[k]["bytes"] / t / 1e9, 1),
                    "tflops": round(work[k]["flops"] / t / 1e12, 2), "roofline": roof_k}
    dom = max(KERNELS, key=lambda k: per_kernel_ms[k])
    t_dom = per_kernel_ms[dom] * 1e-3
    roof = dict(kernel=dom, **roofline_entry(work[dom], t_dom, peaks, "tensor" if dom == "gemm" else "hbm"))
    roof["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json burst)" if peak_src == "measured" else "fallback"
    roof["traffic"] = TRAFFIC.get(dom)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "rows": ROWS, "cols": COLS, "gemv_batch": GEMV_B, "gemm_m": GEMM_M,
                   "weight": "bf16 ~N(0,0.02), 0.1% x20 outliers, seeds 1002/1003; NF4 blocksize 64, "
                             "double quant E4M3 blocks of 256",
                   "l2": f"step inputs rotate over {copies} copies ({copies * per_copy / 1e6:.0f} MB > L2 "
                         f"{l2 / 1e6:.0f} MB); every leg below rotates >= 3x L2 of its own inputs",
                   "parallelism": "replicas" if world > 1 else "single"},
        "roofline": roof,
        "breakdown": breakdown,
        "configs": configs,
        "next": nexts,
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": int(launches),
        "gpu_launches_configs": int(cfg_launches),
        "launch": ("the K timed steps captured in one CUDA graph, launches chained with programmatic dependent "
                   "launch; every per-kernel and per-config figure from one graph of K to 64 launches (about 2 ms) of that call over "
                   "rotating input sets; e2e leg launches eagerly, copies in, library calls and copies out on three "
                   "streams overlapping across steps"),
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


def model_config(args, nf4, synth, dev, time_calls, peaks):
    """config 5: quantize + double quant of all 224 weights of the 8B-shaped stack, then one decode GEMV pass over
    them (one nf4_gemv_stream launch) at batch 1, 4 and 8"""
    import torch
    shapes = model_shapes()
    srcs, qws, bufs = [], [], []
    for layer, p, r, c in shapes:
        srcs.append(synth.normal_weights_device((r, c), synth.layer_seed(layer, p), device=dev))
        nbm = r * c // 64
        packed = torch.empty(r * c // 2, dtype=torch.uint8, device=dev)
        absmax = torch.empty(nbm, dtype=torch.float32, device=dev)
        q = torch.empty(nbm, dtype=torch.uint8, device=dev)
        scale = torch.empty(-(-nbm // 256), dtype=torch.float32, device=dev)
        mean = torch.empty(1, dtype=torch.float32, device=dev)
        bufs.append((packed, absmax, q, scale, mean))
        qws.append(nf4.QuantizedWeight(packed=packed, rows=r, cols=c, absmax_q=q, absmax_scale=scale,
                                       absmax_mean=mean, dq_code=nf4.NF4_DQ_E4M3))
    dq_ws = torch.zeros(nf4._lib.load().nf4_double_quant_many_workspace_bytes(len(shapes)), dtype=torch.uint8, device=dev)
    absmaxes = [b[1] for b in bufs]
    dq_outs = [b[2:5] for b in bufs]

    flat = [s.reshape(-1) for s in srcs]
    q_outs = [b[0:2] for b in bufs]

    def quantize_pass():
        # all 224 weights quantized in one call, then the double quant of all 224 absmax arrays in one call
        nf4.quantize_many(flat, outs=q_outs)
        nf4.double_quant_many(absmaxes, "e4m3", outs=dq_outs, workspace=dq_ws)

    reps = 3
    t_quant = time_calls([quantize_pass], n=reps) * 1e-3
    launches = 3 * reps
    mw = model_work(1)
    out = {"what": "32 layers x (q 4096x4096, k/v 1024x4096, o 4096x4096, gate/up 14336x4096, down 4096x14336) "
                   "bf16 ~N(0,0.02) (device generator, seed 2000 + 7 layer + proj), 6,979,321,856 weights; "
                   f"quantize of all 224 in one nf4_quantize_many call, then E4M3 double quant of all 224 absmax "
                   f"arrays in one nf4_double_quant_many call (3 launches per pass, {reps} passes timed); then "
                   "one decode GEMV pass over all 224 weights as one nf4_gemv_stream launch, inputs for q/k/v, o, "
                   "gate/up and down of every layer ~N(0,1) (seeds 3300 + 10 b + j)",
           "quantize_pass": {"ms": round(t_quant * 1e3, 4), "gelem_s": round(mw["quantize_pass"]["elems"] / t_quant / 1e9, 1),
                             "roofline": roofline_entry(mw["quantize_pass"], t_quant, peaks, "hbm")}}
    del srcs, flat
    torch.cuda.empty_cache()
    for b in GEMV_BATCHES:
        acts = [synth.activations_device((b, c), 3300 + 10 * b + j, device=dev)
                for j, c in enumerate((4096, 4096, 4096, 14336))]
        xs = []
        for _ in range(synth.LLAMA8B_LAYERS):
            xs += [acts[0]] * 3 + [acts[1]] + [acts[2]] * 2 + [acts[3]]
        outs = [torch.empty(b, q.rows, dtype=torch.bfloat16, device=dev) for q in qws]
        # 3.6 GB of codes per pass: every pass reads cold weights without rotation
        t = time_calls([lambda xs=xs, outs=outs: nf4.gemv_stream(qws, xs, outs=outs)]) * 1e-3
        launches += args.steps
        w = model_work(b)["gemv_pass"]
        out[f"gemv_pass_b{b}"] = {"ms": round(t * 1e3, 4), "passes_s": round(1 / t, 1),
                                  "launches_per_pass": 1, "roofline": roofline_entry(w, t, peaks, "hbm")}
    out["_launches"] = launches
    del qws, bufs
    torch.cuda.empty_cache()
    return out


# ncu dram__bytes_read.sum + dram__bytes_write.sum per launch of each kernel at this workload (double quant: its two
# kernels; gemm_lora: the down map and the GEMM), from the captures summarised in profiles/ (ncu flushes the caches
# before each replayed launch, so these are cold-read figures); an entry is removed whenever its kernel changes
# after the capture
TRAFFIC = {"quantize": 33576448, "double_quant": 2161664, "dequantize": 8688896, "gemv": 8681984, "gemm": 10823424,
           "gemm_dx": 10819328, "gemm_lora": 13227264, "gemv_grouped": 13011200}


def oracle_table(args):
    """The CPU oracle per reference config, on all host cores and on one, each on a bounded sample of the config's
    workload (stated per row; rows of a matmul sample are weight rows, all activation rows kept).  Prints one JSON
    object; the figures are a baseline for the tables, not a target."""
    import numpy as np
    import oracle
    from qlora_block_absmax_b200 import synth
    oracle.build()
    cores = oracle.get_threads()
    rng = synth.rng(5)

    def timed(f):
        t0 = time.perf_counter()
        f()
        return time.perf_counter() - t0

    def row(work_bytes, seconds, unit="GB/s", flops=None, elems=None, sample=""):
        d = {"seconds": round(seconds, 4), "gbs": round(work_bytes / seconds / 1e9, 4), "sample": sample}
        if flops:
            d["gflops"] = round(flops / seconds / 1e9, 4)
        if elems:
            d["melem_s"] = round(elems / seconds / 1e6, 3)
        return d

    def both(fn):
        out = {}
        for name, threads, frac in (("all_cores", cores, 1), ("one_core", 1, 8)):
            oracle.set_threads(threads)
            out[name] = fn(frac)
        oracle.set_threads(cores)
        return out

    table = {"cores": cores, "cpu_model": cpu_model()}
    w1 = synth.fp32_1024x1024_weight()

    def cfg1(frac):
        n = w1.size // frac
        p, a = oracle.quantize(w1.reshape(-1)[:n])
        tq = timed(lambda: oracle.quantize(w1.reshape(-1)[:n]))
        td = timed(lambda: oracle.dequantize(p, a, n, 64, "f32"))
        return {"quantize": row(4.5625 * n, tq, elems=n, sample=f"{n} of {w1.size} elements"),
                "dequantize_f32": row(4.5625 * n, td, elems=n, sample=f"{n} of {w1.size} elements")}
    table["1_fp32_1024x1024"] = both(cfg1)
    w2 = synth.bf16_4096x4096_outlier_weight().reshape(-1)

    def cfg2(frac):
        n = w2.size // (4 * frac)
        tq = timed(lambda: oracle.quantize(w2[:n]))
        _, a = oracle.quantize(w2[:n])
        td = timed(lambda: oracle.double_quant(a, 256, oracle.DQ_E4M3))
        return {"quantize": row(2.5625 * n, tq, elems=n, sample=f"first {n} of {w2.size} elements"),
                "double_quant_e4m3": row(5.0 * a.size, td, sample=f"{a.size} absmax values")}
    table["2_bf16_4096x4096_dq"] = both(cfg2)
    cached = {}

    def weight(rows, cols, seed):
        key = (rows, cols, seed)
        if key not in cached:
            w = synth.normal_weights((rows, cols), seed)
            p, a = oracle.quantize(w.reshape(-1))
            q, sc, mu = oracle.double_quant(a, 256, oracle.DQ_E4M3)
            cached[key] = (p, oracle.absmax_reconstruct(q, sc, mu, 256, oracle.DQ_E4M3))
        return cached[key]

    def cfg3(frac):
        out = {}
        for r, c in GEMV_SHAPES:
            p, ah = weight(r, c, 1010)
            for b in (1, 8):
                x = synth.activations((b, c), 1013)
                sub = r // frac
                t = timed(lambda: oracle.matmul(p[:sub * c // 2], ah[:sub * c // 64], sub, c, x))
                wk = gemv_work(sub, c, b)
                out[f"{r}x{c}_b{b}"] = row(wk["bytes"], t, flops=wk["flops"],
                                           sample=f"first {sub} of {r} weight rows, fp64 accumulation")
        return out
    table["3_gemv"] = both(cfg3)

    def cfg4(frac):
        out = {}
        r, c = GEMM_SHAPE
        p, ah = weight(r, c, 1020)
        for m in GEMM_MS:
            sub = max(16, min(r, (r * 64) // m) // frac // 16 * 16)
            x = synth.activations((m, c), 1021 + m)
            t = timed(lambda: oracle.matmul(p[:sub * c // 2], ah[:sub * c // 64], sub, c, x))
            wk = gemm_work(sub, c, m)
            out[f"M{m}"] = row(wk["bytes"], t, flops=wk["flops"],
                               sample=f"first {sub} of {r} weight rows x all {m} activation rows; "
                                      f"the full product scales by {r / sub:.1f}x")
        return out
    table["4_gemm_14336x4096"] = both(cfg4)

    def cfg5(frac):
        # one decoder layer (7 weights), generated on the host; the 32-layer stack is 32x this work
        out = {}
        layer = []
        t_q = 0.0
        for p_i, (name, r, c) in enumerate(synth.LLAMA8B_LAYER):
            sub = r // frac
            w = synth.f32_to_bf16_bits(synth.normal_weights((sub, c), synth.layer_seed(0, p_i)))
            t0 = time.perf_counter()
            p, a = oracle.quantize(w.reshape(-1))
            q, sc, mu = oracle.double_quant(a, 256, oracle.DQ_E4M3)
            t_q += time.perf_counter() - t0
            layer.append((sub, c, p, oracle.absmax_reconstruct(q, sc, mu, 256, oracle.DQ_E4M3)))
        nq = sum(sub * c for sub, c, _, _ in layer)
        out["quantize_layer"] = row(sum(2.5625 * sub * c + 5 * sub * c / 64 for sub, c, _, _ in layer), t_q, elems=nq,
                                    sample=f"layer 0 of 32 ({'all' if frac == 1 else f'1/{frac} of the'} rows of "
                                           f"each of its 7 weights): quantize + E4M3 double quant")
        x = {4096: synth.activations((1, 4096), 3301), 14336: synth.activations((1, 14336), 3304)}
        t_g = sum(timed(lambda sub=sub, c=c, p=p, ah=ah: oracle.matmul(p, ah, sub, c, x[c])) for sub, c, p, ah in layer)
        wb = sum(gemv_work(sub, c, 1)["bytes"] for sub, c, _, _ in layer)
        out["gemv_layer_b1"] = row(wb, t_g, sample="the same layer, batch 1; a model pass is 32 layers")
        return out
    table["5_model_8b"] = both(cfg5)
    print(json.dumps(table), flush=True)


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
    ap.add_argument("--quick", action="store_true", help="skip the whole-model config (5)")
    ap.add_argument("--oracle-table", action="store_true", help="time the CPU oracle per config (1 and all cores)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.oracle_table:
        oracle_table(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
