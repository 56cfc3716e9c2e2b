"""bench.py's algorithmic work per step (the numerators of every throughput and roofline figure), checked on the CPU
against the definitions: each operand read once and each output written once at its stored width."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_step_work_matches_definitions():
    rows, cols, b, m = 4096, 4096, 1, 256
    w = bench.work_per_step(rows, cols, b, m)
    n = rows * cols
    nb = n // 64
    record = n // 2 + nb + 4 * (nb // 256) + 4          # codes + E4M3 codes + second-level scales + mean
    assert w["quantize"] == {"bytes": 2 * n + n // 2 + 4 * nb, "elems": n}
    assert w["double_quant"]["bytes"] == 4 * nb + nb + 4 * (nb // 256) + 4
    assert w["dequantize"]["bytes"] == record + 2 * n
    assert w["gemv"]["bytes"] == record + 2 * b * cols + 2 * b * rows and w["gemv"]["flops"] == 2 * b * n
    assert w["gemm"]["bytes"] == record + 2 * m * cols + 2 * m * rows and w["gemm"]["flops"] == 2 * m * n
    assert w["gemm_dx"]["flops"] == 2 * m * n
    r = bench.LORA_R
    assert w["gemm_lora"]["flops"] == 2 * m * n + 2 * m * r * (rows + cols)
    qkv = sum(rr * cc for rr, cc in bench.QKV_SHAPES)
    assert w["gemv_grouped"]["flops"] == 2 * b * qkv and w["gemv_grouped"]["bound"] == "hbm"
    # the headline sums the five step kernels only; the rows beside the step are reported on their own
    assert set(bench.KERNELS) == {"quantize", "double_quant", "dequantize", "gemv", "gemm"}
    assert not set(bench.KERNELS) & set(bench.NEXT_KERNELS)


def test_replica_throughput_is_whole_job():
    # two replicas, 1 MB per step each, 10 steps in 2.5 ms on the slowest rank -> 8 GB/s
    assert abs(bench.replica_throughput(1e6, 10, 2.5, 2) - 8.0) < 1e-9
