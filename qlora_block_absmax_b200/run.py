"""Run one library call on the benchmark's seeded synthetic inputs, a few times, on cuda:0.

    python -m qlora_block_absmax_b200.run OP [--rows R] [--cols C] [--batch B] [--m M] [--iters N] [--fp4]

OP: quantize | double_quant | dequantize | gemv | gemv_grouped | gemv_stream | gemm | gemm_dx | gemm_lora |
    quantize_many | double_quant_many
Weights: bf16 ~N(0, 0.02) from the device generator (seed 1010), NF4 (or FP4 with --fp4) with E4M3 double quant;
activations bf16 ~N(0, 1) (seed 1013).  gemv_stream runs one decoder layer of the 8B shape (7 weights) in one
launch; gemv_grouped runs q, k, v of that layer (4096, 1024, 1024 x 4096) on one x in one launch;
quantize_many quantizes that layer's 7 weights in one launch and double_quant_many double-quantizes their absmax
arrays in one call.  Useful to look
at one kernel in isolation (for instance under a profiler); prints one line per call
with the device time of the last iteration.
"""
from __future__ import annotations

import argparse

import torch

import qlora_block_absmax_b200 as nf4
from qlora_block_absmax_b200 import synth


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("op", choices=["quantize", "double_quant", "dequantize", "gemv", "gemv_grouped", "gemv_stream",
                                   "gemm", "gemm_dx", "gemm_lora", "quantize_many", "double_quant_many"])
    ap.add_argument("--rows", type=int, default=4096)
    ap.add_argument("--cols", type=int, default=4096)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--m", type=int, default=256)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--fp4", action="store_true")
    a = ap.parse_args()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    qt = "fp4" if a.fp4 else "nf4"
    w = synth.normal_weights_device((a.rows, a.cols), 1010, device=dev)
    qw = nf4.quantize_weight(w, quant_type=qt)
    if a.op == "quantize":
        out = (torch.empty(w.numel() // 2, dtype=torch.uint8, device=dev),
               torch.empty(w.numel() // 64, dtype=torch.float32, device=dev))
        call = lambda: nf4.quantize(w, out=out, quant_type=qt)  # noqa: E731
    elif a.op == "double_quant":
        _, absmax = nf4.quantize(w, quant_type=qt)
        ws = torch.zeros(256, dtype=torch.uint8, device=dev)
        call = lambda: nf4.double_quant(absmax, "e4m3", workspace=ws)  # noqa: E731
    elif a.op == "dequantize":
        out = torch.empty(a.rows, a.cols, dtype=torch.bfloat16, device=dev)
        call = lambda: nf4.dequantize(qw, torch.bfloat16, out=out)  # noqa: E731
    elif a.op == "gemv":
        x = synth.activations_device((a.batch, a.cols), 1013, device=dev)
        call = lambda: nf4.gemv(qw, x)  # noqa: E731
    elif a.op == "gemv_grouped":
        x = synth.activations_device((a.batch, 4096), 1013, device=dev)
        qkv = [nf4.quantize_weight(synth.normal_weights_device((r, 4096), synth.layer_seed(0, p), device=dev),
                                   quant_type=qt) for p, (_, r, _) in enumerate(synth.LLAMA8B_LAYER[:3])]
        call = lambda: nf4.gemv_grouped(qkv, x)  # noqa: E731
    elif a.op in ("quantize_many", "double_quant_many"):
        srcs = [synth.normal_weights_device((r, c), synth.layer_seed(0, p), device=dev).reshape(-1)
                for p, (_, r, c) in enumerate(synth.LLAMA8B_LAYER)]
        outs = nf4.quantize_many(srcs)
        if a.op == "quantize_many":
            call = lambda: nf4.quantize_many(srcs, outs=outs)  # noqa: E731
        else:
            absmaxes = [o[1] for o in outs]
            ws = torch.zeros(nf4._lib.load().nf4_double_quant_many_workspace_bytes(len(srcs)), dtype=torch.uint8,
                             device=dev)
            call = lambda: nf4.double_quant_many(absmaxes, "e4m3", workspace=ws)  # noqa: E731
    elif a.op == "gemv_stream":
        ws, xs = [], []
        acts = [synth.activations_device((a.batch, c), 3300 + j, device=dev) for j, c in enumerate((4096, 14336))]
        for p, (name, r, c) in enumerate(synth.LLAMA8B_LAYER):
            ws.append(nf4.quantize_weight(synth.normal_weights_device((r, c), synth.layer_seed(0, p), device=dev),
                                          quant_type=qt))
            xs.append(acts[1] if name == "down" else acts[0])
        call = lambda: nf4.gemv_stream(ws, xs)  # noqa: E731
    else:
        x = synth.activations_device((a.m, a.cols), 1013, device=dev)
        if a.op == "gemm":
            ws = torch.zeros(max(16, nf4.gemm_workspace_bytes(qw, a.m)), dtype=torch.uint8, device=dev)
            call = lambda: nf4.gemm(qw, x, workspace=ws)  # noqa: E731
        elif a.op == "gemm_dx":
            dy = synth.activations_device((a.m, a.rows), 1014, device=dev)
            ws = torch.zeros(max(16, nf4.gemm_dx_workspace_bytes(qw, a.m)), dtype=torch.uint8, device=dev)
            call = lambda: nf4.gemm_dx(qw, dy, workspace=ws)  # noqa: E731
        else:
            g = torch.Generator(device=dev)
            g.manual_seed(1281)
            down = (torch.randn(16, a.cols, generator=g, device=dev) / a.cols ** 0.5).to(torch.bfloat16)
            up = (torch.randn(a.rows, 16, generator=g, device=dev) * 0.02).to(torch.bfloat16)
            ws = torch.zeros(nf4.gemm_lora_workspace_bytes(qw, a.m), dtype=torch.uint8, device=dev)
            call = lambda: nf4.gemm_lora(qw, x, down, up, 2.0, workspace=ws)  # noqa: E731
    for _ in range(a.iters):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        torch.cuda.synchronize()
    nf4.check_device_error()
    print(f"{a.op} rows={a.rows} cols={a.cols} batch={a.batch} m={a.m} {qt}: {e0.elapsed_time(e1) * 1e3:.2f} us "
          f"(last of {a.iters}, eager)")


if __name__ == "__main__":
    main()
