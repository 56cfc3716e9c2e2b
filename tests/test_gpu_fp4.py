"""FP4 codes (E2M1 / 6 by bit pattern; "bitsandbytes", "Glossary" and "What it is": the other 4-bit format) in
the kernels, against the oracle's FP4 functions: packed codes and absmax bit for bit (including blocks of zeros,
signed zeros, negative maxima, constants, exact levels, exact midpoints and tiny scales), fp32 and bf16
dequantization bit for bit (plain and double-quantized scales), and the GEMV and GEMM within the matmul tolerance
(per output 1e-2 relative, floor 1e-3 * rms)."""
import numpy as np
import pytest
import torch

import oracle
import qlora_block_absmax_b200 as nf4
from qlora_block_absmax_b200 import synth

from tests.test_gpu_parity import check_matmul, dev, dev_bf16, host_bf16_bits

pytestmark = pytest.mark.gpu


def fp4_special_weights(n_blocks: int, seed: int) -> np.ndarray:
    """normal weights with hand-made blocks: zeros, signed zeros, negative max, a constant, exact FP4 levels, exact
    level midpoints, tiny and subnormal scales"""
    w = synth.normal_weights((n_blocks * 64,), seed)
    _, c = oracle.fp4_codebook()
    blocks = w.reshape(-1, 64)
    blocks[0] = 0.0
    blocks[1, ::2] = -0.0
    blocks[1, 1::2] = 0.0
    blocks[2] = -np.abs(blocks[2])
    blocks[3] = np.float32(-0.25)
    blocks[4, :16] = c
    blocks[4, 16:] = c[np.arange(48) % 16] * np.float32(0.5)
    blocks[4, 7] = 1.0
    mags = np.sort(c[:8])
    mids = ((mags[:-1].astype(np.float64) + mags[1:]) / 2).astype(np.float32)
    blocks[5, :7] = mids
    blocks[5, 7:14] = -mids
    blocks[5, 14] = 1.0
    blocks[6] = blocks[6] * np.float32(1e-38)
    blocks[7] = blocks[7] * np.float32(3e-42)
    blocks[8, :] = np.float32(1e-3)
    blocks[8, 0] = np.float32(-1.0)
    return w


@pytest.mark.parametrize("n", [1, 2, 63, 65, 129, 4097, 64 * 1000 + 33])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_fp4_quantize_bit_exact(n, dtype):
    w = synth.normal_weights((n,), 300 + n)
    src = w if dtype == "f32" else synth.f32_to_bf16_bits(w)
    p_ref, a_ref = oracle.fp4_quantize(src)
    t = dev(w) if dtype == "f32" else dev_bf16(src)
    p, a = nf4.quantize(t, quant_type="fp4")
    assert np.array_equal(p.cpu().numpy(), p_ref)
    assert np.array_equal(a.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_fp4_quantize_special_blocks(dtype):
    w = fp4_special_weights(64, 17)
    src = w if dtype == "f32" else synth.f32_to_bf16_bits(w)
    p_ref, a_ref = oracle.fp4_quantize(src)
    p, a = nf4.quantize(dev(w) if dtype == "f32" else dev_bf16(src), quant_type="fp4")
    assert np.array_equal(p.cpu().numpy(), p_ref)
    assert np.array_equal(a.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
    # the all-zero block is all +0 codes; the signed-zero block keeps its signs (pattern 8 for -0)
    assert np.all(p_ref[:32] == 0)


def test_fp4_quantize_reference_configs():
    """the fp32 1024x1024 round-trip weight and the bf16 4096x4096 weight with outliers, in full"""
    w1 = synth.fp32_1024x1024_weight()
    p_ref, a_ref = oracle.fp4_quantize(w1)
    p, a = nf4.quantize(dev(w1), quant_type="fp4")
    assert np.array_equal(p.cpu().numpy(), p_ref) and np.array_equal(a.cpu().numpy(), a_ref)
    deq = nf4.dequantize(nf4.QuantizedWeight(packed=p, rows=1024, cols=1024, absmax=a,
                                             quant_type=nf4.NF4_QUANT_FP4), torch.float32)
    ref = oracle.fp4_dequantize(p_ref, a_ref, w1.size, 64, "f32")
    assert np.array_equal(deq.cpu().numpy().reshape(-1).view(np.uint32), ref.view(np.uint32))
    w2 = synth.bf16_4096x4096_outlier_weight()
    p_ref, a_ref = oracle.fp4_quantize(w2.reshape(-1))
    p, a = nf4.quantize(dev_bf16(w2), quant_type="fp4")
    assert np.array_equal(p.cpu().numpy(), p_ref) and np.array_equal(a.cpu().numpy(), a_ref)


def fp4_pair(rows, cols, seed, use_dq, code="e4m3"):
    w = synth.normal_weights((rows, cols), seed)
    qw = nf4.quantize_weight(dev(w), use_double_quant=use_dq, code=code, quant_type="fp4")
    p_ref, a_ref = oracle.fp4_quantize(w.reshape(-1))
    if use_dq:
        c = oracle.DQ_E4M3 if code == "e4m3" else oracle.DQ_INT8
        q_ref, s_ref, m_ref = oracle.double_quant(a_ref, 256, c)
        a_ref = oracle.absmax_reconstruct(q_ref, s_ref, m_ref, 256, c)
    return qw, p_ref, a_ref


@pytest.mark.parametrize("use_dq,code", [(False, "e4m3"), (True, "e4m3"), (True, "int8")])
@pytest.mark.parametrize("out", ["f32", "bf16"])
@pytest.mark.parametrize("rows,cols", [(1, 1), (3, 21), (37, 129), (128, 640)])
def test_fp4_dequantize_bit_exact(use_dq, code, out, rows, cols):
    qw, p_ref, a_ref = fp4_pair(rows, cols, rows * cols + 5, use_dq, code)
    got = nf4.dequantize(qw, torch.float32 if out == "f32" else torch.bfloat16)
    ref = oracle.fp4_dequantize(p_ref, a_ref, rows * cols, 64, out)
    g = got.cpu().numpy().reshape(-1).view(np.uint32) if out == "f32" else host_bf16_bits(got).reshape(-1)
    assert np.array_equal(g, ref.view(np.uint32) if out == "f32" else ref)


@pytest.mark.parametrize("shape", [(4096, 4096), (14336, 4096), (4096, 14336), (48, 320)])
@pytest.mark.parametrize("batch", [1, 4, 8])
def test_fp4_gemv(shape, batch):
    rows, cols = shape
    qw, p_ref, a_ref = fp4_pair(rows, cols, 1040 + rows // 16 + cols, True)
    x = synth.activations((batch, cols), 1013 + batch)
    check_matmul(nf4.gemv(qw, dev_bf16(x)), oracle.fp4_matmul(p_ref, a_ref, rows, cols, x), f"fp4 gemv {shape} b{batch}")


def test_fp4_gemv_stream_and_mixed_books_rejected():
    pairs = [fp4_pair(r, c, 1060 + i, i % 2 == 0) for i, (r, c) in enumerate(((256, 1024), (64, 4096), (1024, 320)))]
    xs = [synth.activations((2, qw.cols), 1070 + i) for i, (qw, _, _) in enumerate(pairs)]
    ys = nf4.gemv_stream([p[0] for p in pairs], [dev_bf16(x) for x in xs])
    for (qw, p_ref, a_ref), x, y in zip(pairs, xs, ys):
        check_matmul(y, oracle.fp4_matmul(p_ref, a_ref, qw.rows, qw.cols, x), "fp4 stream")
    nf4_w = nf4.quantize_weight(dev(synth.normal_weights((16, 1024), 3)))
    with pytest.raises(nf4.NF4Error):
        nf4.gemv_stream([pairs[0][0], nf4_w], [dev_bf16(xs[0]), dev_bf16(xs[0])])


@pytest.mark.parametrize("m", [1, 16, 33, 64, 65, 256, 1024])
def test_fp4_gemm(m):
    rows, cols = 1024, 4096
    qw, p_ref, a_ref = fp4_pair(rows, cols, 1080, True)
    x = synth.activations((m, cols), 1081 + m)
    check_matmul(nf4.gemm(qw, dev_bf16(x)), oracle.fp4_matmul(p_ref, a_ref, rows, cols, x), f"fp4 gemm m{m}")


def test_fp4_gemm_split_and_plain_scales():
    rows, cols, m = 256, 2048, 300
    qw, p_ref, a_ref = fp4_pair(rows, cols, 1090, False)
    x = synth.activations((m, cols), 1091)
    check_matmul(nf4.gemm(qw, dev_bf16(x)), oracle.fp4_matmul(p_ref, a_ref, rows, cols, x), "fp4 gemm split")
    nf4.check_device_error()
