"""Level-1 block sizes 32, 128 and 256 besides 64 ("bitsandbytes", "How it works" Steps 1-5: one absmax per block of
consecutive elements; pre-quantized checkpoints differ in the block size): quantize (NF4 and FP4, fp32 and bf16
inputs) and dequantize (fp32 and bf16 outputs, plain and double-quantized scales) bit for bit against the oracle,
on sizes with ragged tails; the matmuls reject the other sizes."""
import numpy as np
import pytest
import torch

import oracle
import qlora_block_absmax_b200 as nf4
from qlora_block_absmax_b200 import synth

from tests.test_gpu_parity import dev, dev_bf16

pytestmark = pytest.mark.gpu

SIZES = [1, 31, 33, 127, 129, 257, 4097, 256 * 1000 + 97]


def _oracle_quantize(src, bs, qt):
    return oracle.fp4_quantize(src, bs) if qt == "fp4" else oracle.quantize(src, bs)


def _oracle_dequantize(p, a, n, bs, out, qt):
    return oracle.fp4_dequantize(p, a, n, bs, out) if qt == "fp4" else oracle.dequantize(p, a, n, bs, out)


@pytest.mark.parametrize("bs", [32, 128, 256])
@pytest.mark.parametrize("n", SIZES)
@pytest.mark.parametrize("qt", ["nf4", "fp4"])
def test_quantize_dequantize_blocksizes(bs, n, qt):
    w = synth.normal_weights((n,), 700 + n + bs)
    for dtype in ("f32", "bf16"):
        src = w if dtype == "f32" else synth.f32_to_bf16_bits(w)
        p_ref, a_ref = _oracle_quantize(src, bs, qt)
        p, a = nf4.quantize(dev(w) if dtype == "f32" else dev_bf16(src), blocksize=bs, quant_type=qt)
        assert a.numel() == (n + bs - 1) // bs
        assert np.array_equal(p.cpu().numpy(), p_ref)
        assert np.array_equal(a.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
    qw = nf4.QuantizedWeight(packed=p, rows=1, cols=n, absmax=a, blocksize=bs, quant_type=nf4._QUANT_TYPES[qt])
    for out, tdt, view in (("f32", torch.float32, np.uint32), ("bf16", torch.bfloat16, np.uint16)):
        got = nf4.dequantize(qw, tdt).cpu()
        got = got.view(torch.int16).numpy().view(np.uint16) if out == "bf16" else got.numpy().view(np.uint32)
        ref = _oracle_dequantize(p_ref, a_ref, n, bs, out, qt)
        assert np.array_equal(got.reshape(-1), ref.view(view))


@pytest.mark.parametrize("bs", [32, 128, 256])
@pytest.mark.parametrize("code", ["e4m3", "int8"])
def test_dequantize_double_quant_blocksizes(bs, code):
    """double-quantized scales of a [1000, 1000 + 3]-shaped weight: the record is the oracle's, the output bit exact"""
    rows, cols = 1000, 1003
    w = synth.normal_weights((rows, cols), 900 + bs)
    p_ref, a_ref = oracle.quantize(w.reshape(-1), bs)
    dq = oracle.DQ_E4M3 if code == "e4m3" else oracle.DQ_INT8
    q, scale, mean = oracle.double_quant(a_ref, 256, dq)
    a_hat = oracle.absmax_reconstruct(q, scale, mean, 256, dq)
    d = torch.device("cuda", 0)
    qw = nf4.QuantizedWeight(packed=torch.from_numpy(p_ref).to(d), rows=rows, cols=cols,
                             absmax_q=torch.from_numpy(q).to(d), absmax_scale=torch.from_numpy(scale).to(d),
                             absmax_mean=torch.tensor([mean], dtype=torch.float32, device=d),
                             dq_code=nf4._DQ_CODES[code], blocksize=bs)
    for out, tdt, view in (("f32", torch.float32, np.uint32), ("bf16", torch.bfloat16, np.uint16)):
        got = nf4.dequantize(qw, tdt).cpu()
        got = got.view(torch.int16).numpy().view(np.uint16) if out == "bf16" else got.numpy().view(np.uint32)
        ref = oracle.dequantize(p_ref, a_hat, rows * cols, bs, out)
        assert np.array_equal(got.reshape(-1), ref.view(view))


@pytest.mark.parametrize("bs", [32, 128])
def test_matmuls_reject_other_blocksizes(bs):
    w = dev(synth.normal_weights((64, 256), 5))
    qw = nf4.quantize_weight(w, use_double_quant=False, blocksize=bs)
    x = torch.zeros(1, 256, dtype=torch.bfloat16, device=w.device)
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        nf4.gemv(qw, x)
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        nf4.gemm(qw, torch.zeros(16, 256, dtype=torch.bfloat16, device=w.device))
