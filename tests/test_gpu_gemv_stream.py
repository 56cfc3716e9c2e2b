"""The multi-weight decode GEMV (nf4_gemv_stream): many weights, each with its own input and output, in one
persistent launch.  Every output must match the fp64 oracle within the matmul tolerance (per-output 1e-2, floor
1e-3 * rms) and nf4_gemv's output for the same weight within the same tolerance (the two kernels add the fp32
partials in different orders); repeated launches give identical bits."""
import numpy as np
import pytest
import torch

import oracle
import qlora_block_absmax_b200 as nf4
from qlora_block_absmax_b200 import synth

from tests.test_gpu_parity import check_matmul, dev, dev_bf16, quantized_pair

pytestmark = pytest.mark.gpu


def run_and_check(specs, batch, seed, compare_single=True):
    """specs: list of (rows, cols, use_dq, code); every weight gets its own x"""
    pairs = [quantized_pair(r, c, seed + 13 * i + r // 16 + c, dq, code) for i, (r, c, dq, code) in enumerate(specs)]
    xs = [synth.activations((batch, c), seed + 1000 + i) for i, (_, c, _, _) in enumerate(specs)]
    xd = [dev_bf16(x) for x in xs]
    ys = nf4.gemv_stream([p[0] for p in pairs], xd)
    again = nf4.gemv_stream([p[0] for p in pairs], xd)
    nf4.check_device_error()
    for (qw, p_ref, a_ref), x, y, y2, s in zip(pairs, xs, ys, again, specs):
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16)), f"repeat differs {s}"
        ref = oracle.matmul(p_ref, a_ref, qw.rows, qw.cols, x)
        check_matmul(y, ref, f"stream {s} b{batch}")
        if compare_single:
            check_matmul(nf4.gemv(qw, dev_bf16(x)), ref, f"gemv {s} b{batch}")


@pytest.mark.parametrize("batch", [1, 3, 8])
def test_gemv_stream_mixed_weights(batch):
    """shapes, scale kinds and ragged rows mixed in one launch: a single tile, one 64-column block (one step:
    seven of a team's eight warps idle), ragged last steps (320, 4160 columns), several tiles per team"""
    specs = [(16, 64, True, "e4m3"), (48, 320, False, "e4m3"), (128, 4160, True, "int8"), (1024, 4096, True, "e4m3"),
             (16, 1024, False, "e4m3"), (256, 1024, True, "int8"), (32, 14336, True, "e4m3"), (512, 512, True, "e4m3")]
    run_and_check(specs, batch, 400 + batch)


def test_gemv_stream_many_small_weights():
    """the most weights one launch takes (256), each tiny, so items change within every team's tile sequence"""
    specs = [(16 * (1 + i % 3), 64 * (1 + i % 5), i % 2 == 0, "e4m3" if i % 4 else "int8") for i in range(256)]
    run_and_check(specs, 2, 600, compare_single=False)


def test_gemv_stream_rejects_more_than_max():
    qw, _, _ = quantized_pair(16, 64, 1, True)
    x = dev_bf16(synth.activations((1, 64), 2))
    with pytest.raises(nf4.NF4Error):
        nf4.gemv_stream([qw] * 257, [x] * 257)


@pytest.mark.parametrize("batch", [1, 4, 8])
def test_gemv_stream_decoder_layer(batch):
    """the seven projections of one 8B-shaped decoder layer in one launch, on the four inputs a decoder reads
    (q/k/v share one, o its own, gate/up share one, down its own); outputs sampled against the oracle"""
    shapes = synth.LLAMA8B_LAYER
    ws, srcs = [], []
    for p, (name, rows, cols) in enumerate(shapes):
        w = synth.normal_weights_device((rows, cols), synth.layer_seed(5, p))
        ws.append(nf4.quantize_weight(w, use_double_quant=True, code="e4m3"))
        srcs.append(w.view(torch.int16).cpu().numpy().view(np.uint16))
    x_attn = synth.activations_device((batch, 4096), 3200 + batch)
    x_o = synth.activations_device((batch, 4096), 3210 + batch)
    x_mlp = synth.activations_device((batch, 4096), 3220 + batch)
    x_down = synth.activations_device((batch, 14336), 3230 + batch)
    xs = [x_attn, x_attn, x_attn, x_o, x_mlp, x_mlp, x_down]
    ys = nf4.gemv_stream(ws, xs)
    nf4.check_device_error()
    r = synth.rng(91 + batch)
    for (name, rows, cols), qw, src, x, y in zip(shapes, ws, srcs, xs, ys):
        w32 = synth.bf16_bits_to_f32(src.reshape(-1))
        p_ref, a_ref = oracle.quantize(w32)
        q_ref, s_ref, m_ref = oracle.double_quant(a_ref, 256, oracle.DQ_E4M3)
        a_hat = oracle.absmax_reconstruct(q_ref, s_ref, m_ref, 256, oracle.DQ_E4M3)
        xb = x.view(torch.int16).cpu().numpy().view(np.uint16)
        bs, ns = r.integers(0, batch, 512), r.integers(0, rows, 512)
        ref = oracle.matmul_sampled(p_ref, a_hat, rows, cols, xb, bs, ns)
        full_row = oracle.matmul(p_ref, a_hat, rows, cols, xb[:1])
        rms = np.sqrt(np.mean(full_row ** 2))
        got = y.float().cpu().numpy().astype(np.float64)[bs, ns]
        bad = np.abs(got - ref) > 1e-2 * np.maximum(np.abs(ref), 1e-3 * rms)
        assert not bad.any(), (name, int(bad.sum()))
