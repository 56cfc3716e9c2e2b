"""Every output of the products the benchmark times on its own workload -- the bf16 4096x4096 weight with 0.1%
x20 outliers (seeds 1002/1003) quantized to NF4 with E4M3 double quant, M = 256 activation rows -- against the
fp64 oracle, within the matmul tolerance (per output 1e-2 relative, floor 1e-3 * rms): the forward GEMM
(X seed 1277), the input gradient (dY seed 1279) and the GEMM with the r = 16, alpha = 32 adapter (down/up seeds
1281/1282), plus the batch-1 GEMV (x seed 1013)."""
import numpy as np
import pytest

import oracle
import qlora_block_absmax_b200 as nf4
from qlora_block_absmax_b200 import synth

from tests.test_gpu_parity import check_matmul, dev_bf16

pytestmark = pytest.mark.gpu

ROWS, COLS, M, R = 4096, 4096, 256, 16


@pytest.fixture(scope="module")
def bench_weight():
    w_bits = synth.bf16_4096x4096_outlier_weight()
    qw = nf4.quantize_weight(dev_bf16(w_bits), use_double_quant=True, code="e4m3")
    p_ref, a_ref = oracle.quantize(synth.bf16_bits_to_f32(w_bits).reshape(-1))
    q_ref, s_ref, m_ref = oracle.double_quant(a_ref, 256, oracle.DQ_E4M3)
    assert np.array_equal(qw.packed.cpu().numpy(), p_ref)
    assert np.array_equal(qw.absmax_q.cpu().numpy(), q_ref)
    return qw, p_ref, oracle.absmax_reconstruct(q_ref, s_ref, m_ref, 256, oracle.DQ_E4M3)


def test_bench_gemm_every_output(bench_weight):
    qw, p_ref, a_hat = bench_weight
    x = synth.activations((M, COLS), 1277)
    check_matmul(nf4.gemm(qw, dev_bf16(x)), oracle.matmul(p_ref, a_hat, ROWS, COLS, x), "bench gemm")


def test_bench_gemm_dx_every_output(bench_weight):
    qw, p_ref, a_hat = bench_weight
    dy = synth.activations((M, ROWS), 1279)
    check_matmul(nf4.gemm_dx(qw, dev_bf16(dy)), oracle.matmul_dx(p_ref, a_hat, ROWS, COLS, dy), "bench gemm_dx")


def test_bench_gemm_lora_every_output(bench_weight):
    qw, p_ref, a_hat = bench_weight
    x = synth.activations((M, COLS), 1277)
    down = synth.f32_to_bf16_bits((synth.rng(1281).standard_normal((R, COLS)) / np.sqrt(COLS)).astype(np.float32))
    up = synth.f32_to_bf16_bits((synth.rng(1282).standard_normal((ROWS, R)) * 0.02).astype(np.float32))
    y = nf4.gemm_lora(qw, dev_bf16(x), dev_bf16(down), dev_bf16(up), 2.0)
    check_matmul(y, oracle.matmul_lora(p_ref, a_hat, ROWS, COLS, x, down, up, R, 2.0), "bench gemm_lora")


def test_bench_gemv_every_output(bench_weight):
    qw, p_ref, a_hat = bench_weight
    x = synth.activations((1, COLS), 1013)
    check_matmul(nf4.gemv(qw, dev_bf16(x)), oracle.matmul(p_ref, a_hat, ROWS, COLS, x), "bench gemv")
