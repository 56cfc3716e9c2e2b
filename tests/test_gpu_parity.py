"""Parity of the CUDA library (through its C ABI) with the CPU oracle.

Bit-exact: packed codes, fp32 absmax, double-quant codes/scales/mean, fp32 and
bf16 dequantization.  GEMV/GEMM outputs: per-output relative error <= 1e-2
against the fp64-accumulated oracle, with a floor of 1e-3 * rms(y_ref) on the
denominator (outputs whose exact value is near zero cannot be judged
relatively; fp32 accumulation alone gives errors of ~1e-6 * rms there).
"""
import numpy as np
import pytest
import torch

import oracle
import qlora_block_absmax_b200 as nf4
from qlora_block_absmax_b200 import synth

pytestmark = pytest.mark.gpu

REL_TOL = 1e-2
FLOOR = 1e-3


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return dev(bits.view(np.int16)).view(torch.bfloat16)


def host_bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def near_threshold_count(w_f32: np.ndarray, absmax: np.ndarray) -> int:
    """elements whose normalised value lies within 1e-6 of a code midpoint"""
    _, c = oracle.codebook()
    mids = (c[:-1].astype(np.float64) + c[1:]) / 2
    a = np.repeat(absmax, 64)[:w_f32.size].astype(np.float64)
    x = np.divide(w_f32.astype(np.float64), a, out=np.zeros_like(a), where=a > 0)
    return int((np.abs(x[:, None] - mids[None, :]) <= 1e-6).any(axis=1).sum())


def check_matmul(y_gpu: torch.Tensor, y_ref: np.ndarray, what: str):
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    rms = np.sqrt(np.mean(y_ref ** 2)) if y_ref.size else 0.0
    denom = np.maximum(np.abs(y_ref), FLOOR * rms)
    err = np.abs(y - y_ref)
    bad = err > REL_TOL * denom
    floored = int((np.abs(y_ref) < FLOOR * rms).sum())
    assert not bad.any(), (f"{what}: {bad.sum()} of {y.size} outputs beyond 1e-2 (max rel "
                           f"{(err / np.maximum(denom, 1e-300)).max():.3e}, floored {floored})")
    return float((err / np.maximum(denom, 1e-300)).max()), floored


def special_weights(n_blocks: int, seed: int) -> np.ndarray:
    """normal weights with hand-made blocks: zeros, signed zeros, negative max,
    constants, exact code values, values on thresholds, tiny (subnormal) scales"""
    w = synth.normal_weights((n_blocks * 64,), seed)
    _, c = oracle.codebook()
    blocks = w.reshape(-1, 64)
    blocks[0] = 0.0
    blocks[1, ::2] = -0.0
    blocks[1, 1::2] = 0.0
    blocks[2] = -np.abs(blocks[2])
    blocks[3] = np.float32(0.25)
    blocks[4, :16] = c
    blocks[4, 16:] = c[np.arange(48) % 16] * np.float32(0.5)
    mids = np.array([(float(c[i]) + float(c[i + 1])) / 2 for i in range(15)], np.float32)
    blocks[5, :15] = mids
    blocks[5, 15] = 1.0
    blocks[6] = blocks[6] * np.float32(1e-38)     # tiny scale: exact-division path
    blocks[7] = blocks[7] * np.float32(3e-42)     # subnormal scale
    return w


# --------------------------------------------------------------------------- quantize

@pytest.mark.parametrize("n", [1, 2, 63, 64, 65, 127, 129, 4097, 64 * 1000 + 33])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quantize_bit_exact_small(n, dtype):
    w = synth.normal_weights((n,), 7000 + n)
    if dtype == "bf16":
        bits = synth.f32_to_bf16_bits(w)
        p_ref, a_ref = oracle.quantize(bits)
        p, a = nf4.quantize(dev_bf16(bits))
    else:
        p_ref, a_ref = oracle.quantize(w)
        p, a = nf4.quantize(dev(w))
    assert np.array_equal(a.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
    assert np.array_equal(p.cpu().numpy(), p_ref)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quantize_special_blocks(dtype):
    w = special_weights(40, 77)
    if dtype == "bf16":
        bits = synth.f32_to_bf16_bits(w)
        p_ref, a_ref = oracle.quantize(bits)
        p, a = nf4.quantize(dev_bf16(bits))
    else:
        p_ref, a_ref = oracle.quantize(w)
        p, a = nf4.quantize(dev(w))
    assert np.array_equal(a.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
    assert np.array_equal(p.cpu().numpy(), p_ref)


def test_quantize_fp32_1024x1024_roundtrip():
    """fp32 1024x1024 ~N(0,0.02): codes, absmax, fp32 dequantization and
    re-quantization all bit-exact."""
    w = synth.fp32_1024x1024_weight().reshape(-1)
    p_ref, a_ref = oracle.quantize(w)
    p, a = nf4.quantize(dev(w))
    assert np.array_equal(p.cpu().numpy(), p_ref)
    assert np.array_equal(a.cpu().numpy(), a_ref)
    qw = nf4.QuantizedWeight(packed=p, rows=1024, cols=1024, absmax=a)
    wh = nf4.dequantize(qw, torch.float32)
    wh_ref = oracle.dequantize(p_ref, a_ref, w.size)
    assert np.array_equal(wh.cpu().numpy().reshape(-1).view(np.uint32), wh_ref.view(np.uint32))
    p2, a2 = nf4.quantize(wh.reshape(-1))
    assert np.array_equal(p2.cpu().numpy(), p_ref) and np.array_equal(a2.cpu().numpy(), a_ref)
    print(f"fp32 1024x1024: near-midpoint elements {near_threshold_count(w, a_ref)}")


def test_quantize_bf16_4096x4096_outliers():
    bits = synth.bf16_4096x4096_outlier_weight().reshape(-1)
    p_ref, a_ref = oracle.quantize(bits)
    p, a = nf4.quantize(dev_bf16(bits))
    assert np.array_equal(a.cpu().numpy(), a_ref)
    assert np.array_equal(p.cpu().numpy(), p_ref)
    print(f"bf16 4096x4096: near-midpoint elements {near_threshold_count(synth.bf16_bits_to_f32(bits), a_ref)}")


# --------------------------------------------------------------------------- double quant

def dq_cases():
    r = synth.rng(99)
    _, a2 = oracle.quantize(synth.bf16_4096x4096_outlier_weight().reshape(-1))
    return {
        "bf16_4096_outliers": a2,
        "one": np.array([0.3], np.float32),
        "255": np.abs(r.standard_normal(255)).astype(np.float32),
        "257": np.abs(r.standard_normal(257)).astype(np.float32),
        "constant": np.full(700, 0.0625, np.float32),
        "wide": (np.abs(r.standard_normal(3000)) * np.exp(r.uniform(-80, 80, 3000))).astype(np.float32),
        "signed": r.standard_normal(1000).astype(np.float32),
        "zeros_and_tiny": np.concatenate([np.zeros(300, np.float32), np.full(212, 1e-40, np.float32)]),
        # more than 64 values per thread of the sum kernel, magnitudes spread over ~90 binades, some negative
        "big_mixed": (np.abs(r.standard_normal(6_000_001)) * np.exp(r.uniform(-30, 30, 6_000_001))
                      * np.where(r.uniform(0, 1, 6_000_001) < 0.05, -1, 1)).astype(np.float32),
    }


@pytest.mark.parametrize("case", list(dq_cases().keys()))
@pytest.mark.parametrize("code", ["e4m3", "int8"])
def test_double_quant_bit_exact(case, code):
    a = dq_cases()[case]
    c = oracle.DQ_E4M3 if code == "e4m3" else oracle.DQ_INT8
    q_ref, s_ref, m_ref = oracle.double_quant(a, 256, c)
    q, s, m = nf4.double_quant(dev(a), code)
    assert np.float32(m.item()).view(np.uint32) == np.float32(m_ref).view(np.uint32)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_double_quant_workspace_reused():
    """one workspace, zeroed once, across calls of different sizes (different grids) and both codes:
    every call leaves its barrier and exact-sum buffers ready for the next, so each result is exact"""
    cases = dq_cases()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    for name, code in [("bf16_4096_outliers", "e4m3"), ("one", "int8"), ("wide", "e4m3"), ("257", "int8"),
                       ("bf16_4096_outliers", "int8"), ("signed", "e4m3"), ("zeros_and_tiny", "e4m3"), ("bf16_4096_outliers", "e4m3")]:
        a = cases[name]
        c = oracle.DQ_E4M3 if code == "e4m3" else oracle.DQ_INT8
        q_ref, s_ref, m_ref = oracle.double_quant(a, 256, c)
        q, s, m = nf4.double_quant(dev(a), code, workspace=ws)
        assert np.float32(m.item()).view(np.uint32) == np.float32(m_ref).view(np.uint32), name
        assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32)), name
        assert np.array_equal(q.cpu().numpy(), q_ref), name
    nf4.check_device_error()


# --------------------------------------------------------------------------- dequantize

@pytest.mark.parametrize("use_dq,code", [(False, "e4m3"), (True, "e4m3"), (True, "int8")])
@pytest.mark.parametrize("out", ["f32", "bf16"])
@pytest.mark.parametrize("rows,cols", [(1, 1), (3, 21), (16, 64), (37, 129), (128, 640)])
def test_dequantize_bit_exact(use_dq, code, out, rows, cols):
    w = special_weights((rows * cols + 63) // 64 + 8, 5 + rows)[:rows * cols].reshape(rows, cols)
    qw = nf4.quantize_weight(dev(w), use_double_quant=use_dq, code=code)
    p_ref, a_ref = oracle.quantize(w.reshape(-1))
    if use_dq:
        c = oracle.DQ_E4M3 if code == "e4m3" else oracle.DQ_INT8
        q_ref, s_ref, m_ref = oracle.double_quant(a_ref, 256, c)
        a_ref = oracle.absmax_reconstruct(q_ref, s_ref, m_ref, 256, c)
    ref = oracle.dequantize(p_ref, a_ref, rows * cols, 64, out)
    got = nf4.dequantize(qw, torch.float32 if out == "f32" else torch.bfloat16)
    if out == "f32":
        assert np.array_equal(got.cpu().numpy().reshape(-1).view(np.uint32), ref.view(np.uint32))
    else:
        assert np.array_equal(host_bf16_bits(got).reshape(-1), ref)


def test_dequantize_bf16_4096x4096_double_quant():
    bits = synth.bf16_4096x4096_outlier_weight()
    qw = nf4.quantize_weight(dev_bf16(bits), use_double_quant=True, code="e4m3")
    p_ref, a_ref = oracle.quantize(bits.reshape(-1))
    q_ref, s_ref, m_ref = oracle.double_quant(a_ref, 256, oracle.DQ_E4M3)
    ah = oracle.absmax_reconstruct(q_ref, s_ref, m_ref, 256, oracle.DQ_E4M3)
    ref = oracle.dequantize(p_ref, ah, bits.size, 64, "bf16")
    got = nf4.dequantize(qw, torch.bfloat16)
    assert np.array_equal(host_bf16_bits(got).reshape(-1), ref)


# --------------------------------------------------------------------------- matmul

def quantized_pair(rows, cols, seed, use_dq, code="e4m3"):
    w = synth.normal_weights((rows, cols), seed)
    qw = nf4.quantize_weight(dev(w), use_double_quant=use_dq, code=code)
    p_ref, a_ref = oracle.quantize(w.reshape(-1))
    if use_dq:
        c = oracle.DQ_E4M3 if code == "e4m3" else oracle.DQ_INT8
        q_ref, s_ref, m_ref = oracle.double_quant(a_ref, 256, c)
        a_ref = oracle.absmax_reconstruct(q_ref, s_ref, m_ref, 256, c)
    return qw, p_ref, a_ref


@pytest.mark.parametrize("rows,cols", [(16, 64), (16, 192), (48, 320), (128, 256), (256, 4160)])
@pytest.mark.parametrize("batch", [1, 3, 8])
@pytest.mark.parametrize("use_dq", [False, True])
def test_gemv_small(rows, cols, batch, use_dq):
    qw, p_ref, a_ref = quantized_pair(rows, cols, rows + cols + batch, use_dq)
    x = synth.activations((batch, cols), 31 + batch)
    y = nf4.gemv(qw, dev_bf16(x))
    check_matmul(y, oracle.matmul(p_ref, a_ref, rows, cols, x), f"gemv {rows}x{cols} b{batch}")


@pytest.mark.parametrize("shape", [(4096, 4096), (14336, 4096), (4096, 14336), (1024, 4096)])
@pytest.mark.parametrize("batch", [1, 4, 8])
def test_gemv_llama8b_shapes(shape, batch):
    rows, cols = shape
    qw, p_ref, a_ref = quantized_pair(rows, cols, 1010 + rows // 1024 + cols // 1024, True)
    x = synth.activations((batch, cols), 1013)
    y = nf4.gemv(qw, dev_bf16(x))
    mx, floored = check_matmul(y, oracle.matmul(p_ref, a_ref, rows, cols, x), f"gemv {shape} b{batch}")
    print(f"gemv {shape} b{batch}: max floored-rel err {mx:.2e}, floored {floored}")


def test_gemv_one_hot_pins_bit_exact():
    """one-hot activations read single weights back: the decode GEMV (batch <= 8) and the skinny
    tensor-core path (9 <= m <= 64) both return the dequantized bf16 weight bf16_rn(code * a^) bit for bit"""
    rows, cols = 128, 256
    qw, p_ref, a_ref = quantized_pair(rows, cols, 3, True)
    wc = oracle.dequantize(p_ref, a_ref, rows * cols, 64, "bf16").reshape(rows, cols)
    ks = [0, 1, 63, 64, 130, 255, 7, 200, 31, 32, 127, 128, 191, 192, 254, 100]
    x = synth.f32_to_bf16_bits(np.eye(cols, dtype=np.float32)[ks])
    y16 = nf4.gemm(qw, dev_bf16(x))
    assert np.array_equal(host_bf16_bits(y16), wc[:, ks].T)
    y8 = nf4.gemv(qw, dev_bf16(x[:8]))
    assert np.array_equal(host_bf16_bits(y8), wc[:, ks[:8]].T)


# GEMV shapes around the grid's edges: a single 16-row tile; tiles fewer than the SMs; many thin tiles
# (64 or 128 columns); tiles that leave a partial wave; long rows with a ragged last step (cols = 4160).
@pytest.mark.parametrize("rows,cols", [(16, 64), (32, 1024), (65536, 64), (80000, 128), (4096, 4096),
                                       (14336, 4096), (2048, 4160)])
@pytest.mark.parametrize("batch,use_dq,code", [(1, True, "e4m3"), (8, True, "int8"), (5, False, "e4m3")])
def test_gemv_grid_shapes(rows, cols, batch, use_dq, code):
    qw, p_ref, a_ref = quantized_pair(rows, cols, 7 + rows // 16 + cols, use_dq, code)
    x = synth.activations((batch, cols), 77 + batch)
    y1 = nf4.gemv(qw, dev_bf16(x))
    y2 = nf4.gemv(qw, dev_bf16(x))  # same call again: same bits
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    check_matmul(y1, oracle.matmul(p_ref, a_ref, rows, cols, x), f"gemv {rows}x{cols} b{batch}")
    nf4.check_device_error()


def test_gemv_unaligned_scale_codes():
    """double-quant codes starting at an odd address (the record's q array is not 4-byte aligned)"""
    rows, cols = 512, 1536
    qw, p_ref, a_ref = quantized_pair(rows, cols, 21, True)
    q_off = torch.zeros(qw.absmax_q.numel() + 3, dtype=torch.uint8, device="cuda")
    q_off[1:1 + qw.absmax_q.numel()] = qw.absmax_q
    qw2 = nf4.QuantizedWeight(packed=qw.packed, rows=rows, cols=cols, absmax_q=q_off[1:1 + qw.absmax_q.numel()],
                              absmax_scale=qw.absmax_scale, absmax_mean=qw.absmax_mean, dq_code=qw.dq_code)
    assert qw2.absmax_q.data_ptr() % 4 == 1
    x = synth.activations((3, cols), 5)
    y = nf4.gemv(qw2, dev_bf16(x))
    assert torch.equal(y.view(torch.int16), nf4.gemv(qw, dev_bf16(x)).view(torch.int16))
    check_matmul(y, oracle.matmul(p_ref, a_ref, rows, cols, x), "gemv unaligned q")


def test_gemv_zero_codes_give_zero():
    rows, cols = 32, 128
    p = torch.full((rows * cols // 2,), 0x77, dtype=torch.uint8, device="cuda")
    a = torch.rand(rows * cols // 64, device="cuda") + 0.5
    qw = nf4.QuantizedWeight(packed=p, rows=rows, cols=cols, absmax=a)
    x = dev_bf16(synth.activations((5, cols), 4))
    y = nf4.gemv(qw, x)
    assert torch.all(y == 0)


@pytest.mark.parametrize("m", [1, 9, 16, 33, 64, 65, 128, 200, 256])
def test_gemm_small(m):
    rows, cols = 256, 512
    qw, p_ref, a_ref = quantized_pair(rows, cols, 41 + m, True)
    x = synth.activations((m, cols), 42 + m)
    y = nf4.gemm(qw, dev_bf16(x))
    check_matmul(y, oracle.matmul(p_ref, a_ref, rows, cols, x), f"gemm m{m}")


@pytest.mark.parametrize("m", [16, 64, 256, 1024, 4096])
def test_gemm_14336x4096_sampled(m):
    """W 14336x4096 NF4+DQ, X [m, 4096]: 2048 sampled outputs against the oracle,
    plus every output of the first activation row."""
    rows, cols = 14336, 4096
    qw, p_ref, a_ref = quantized_pair(rows, cols, 1020, True)
    x = synth.activations((m, cols), 1021 + m)
    y = nf4.gemm(qw, dev_bf16(x))
    r = synth.rng(5 + m)
    bs = r.integers(0, m, 2048)
    ns = r.integers(0, rows, 2048)
    ref = oracle.matmul_sampled(p_ref, a_ref, rows, cols, x, bs, ns)
    yh = y.float().cpu().numpy().astype(np.float64)
    full_row = oracle.matmul(p_ref, a_ref, rows, cols, x[:1])
    rms = np.sqrt(np.mean(full_row ** 2))
    got = yh[bs, ns]
    assert np.all(np.abs(got - ref) <= REL_TOL * np.maximum(np.abs(ref), FLOOR * rms))
    check_matmul(y[:1], full_row, f"gemm m{m} row 0")


@pytest.mark.parametrize("m", [65, 200, 256, 300])
def test_gemm_split_k(m):
    """few output tiles: K is split across CTAs and the fp32 partials are
    added in split order"""
    rows, cols = 256, 2048
    qw, p_ref, a_ref = quantized_pair(rows, cols, 61 + m, True)
    x = synth.activations((m, cols), 62 + m)
    y = nf4.gemm(qw, dev_bf16(x))
    check_matmul(y, oracle.matmul(p_ref, a_ref, rows, cols, x), f"gemm split m{m}")


def test_gemm_deterministic_and_bench_shape():
    """4096 x 4096 weight, M = 256 (split-K path), the step's own product: bit-identical across calls and every one
    of the 1,048,576 outputs within tolerance of the oracle"""
    rows, cols, m = 4096, 4096, 256
    qw, p_ref, a_ref = quantized_pair(rows, cols, 1002, True)
    x = synth.activations((m, cols), 1277)
    y1 = nf4.gemm(qw, dev_bf16(x))
    y2 = nf4.gemm(qw, dev_bf16(x))
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    check_matmul(y1, oracle.matmul(p_ref, a_ref, rows, cols, x), "gemm 4096x4096 m256 in full")


def test_gemm_dx_bench_shape_in_full():
    """dX = dY . Wc for the 4096 x 4096 weight at M = 256 (split-K path), every one of the 1,048,576 outputs within
    tolerance of the oracle"""
    rows, cols, m = 4096, 4096, 256
    qw, p_ref, a_ref = quantized_pair(rows, cols, 1003, True)
    dy = synth.activations((m, rows), 1279)
    dx = nf4.gemm_dx(qw, dev_bf16(dy))
    check_matmul(dx, oracle.matmul_dx(p_ref, a_ref, rows, cols, dy), "dx 4096x4096 m256 in full")


@pytest.mark.parametrize("rows,m", [(14336, 1024), (4096, 4096), (14336, 256)])
def test_gemm_repeatable_many_tiles(rows, m):
    """Several output tiles per CTA (the persistent grid cycles its rings many times): ten identical calls
    give identical bits.  A slot refilled by TMA before the producer warps' reads of it were ordered, or a
    TMEM read used before it landed, shows up here as a few weight rows differing between calls."""
    cols = 4096
    w = synth.normal_weights((rows, cols), 2024)
    qw = nf4.quantize_weight(dev(w))
    x = dev_bf16(synth.activations((m, cols), 2025))
    ws = torch.zeros(max(nf4.gemm_workspace_bytes(qw, m), 16), dtype=torch.uint8, device="cuda")
    ref = nf4.gemm(qw, x, workspace=ws).view(torch.int16).clone()
    for _ in range(10):
        assert torch.equal(nf4.gemm(qw, x, workspace=ws).view(torch.int16), ref)
    nf4.check_device_error()


@pytest.mark.parametrize("cols", [320, 1024, 4096])
@pytest.mark.parametrize("use_dq", [False, True])
def test_gemm_scale_paths(cols, use_dq):
    """plain fp32 and double-quantized scales, with scale rows that are (1024,
    4096) and are not (320) whole 16-byte units"""
    rows, m = 128, 160
    qw, p_ref, a_ref = quantized_pair(rows, cols, 71 + cols, use_dq)
    x = synth.activations((m, cols), 72 + cols)
    y = nf4.gemm(qw, dev_bf16(x))
    check_matmul(y, oracle.matmul(p_ref, a_ref, rows, cols, x), f"gemm cols{cols} dq{use_dq}")


# --------------------------------------------------------------------------- grouped GEMV (several weights, one input)

@pytest.mark.parametrize("batch", [1, 4, 8])
def test_gemv_grouped_qkv_matches_separate_and_oracle(batch):
    """the q, k, v projections of one 8B-shaped layer (4096, 1024, 1024 rows x 4096) in one launch: each output
    is bit-identical to its own nf4_gemv call (the same per-tile arithmetic) and within the matmul tolerance of
    the oracle"""
    cols = 4096
    pairs = [quantized_pair(rows, cols, 180 + i, True) for i, rows in enumerate((4096, 1024, 1024))]
    x = synth.activations((batch, cols), 183 + batch)
    xd = dev_bf16(x)
    ys = nf4.gemv_grouped([p[0] for p in pairs], xd)
    for (qw, p_ref, a_ref), y in zip(pairs, ys):
        assert torch.equal(y.view(torch.int16), nf4.gemv(qw, xd).view(torch.int16))
        check_matmul(y, oracle.matmul(p_ref, a_ref, qw.rows, cols, x), f"grouped {qw.rows} b{batch}")


@pytest.mark.parametrize("rows_list,use_dq", [((16,), True), ((48, 16, 64, 32), True), ((14336, 14336), True),
                                              ((128, 4096, 16), False)])
def test_gemv_grouped_shapes(rows_list, use_dq):
    """one to four weights, single-tile and mixed sizes, plain and double-quantized scales (each weight
    quantized with its own seed: its own mean and scales)"""
    cols = 1024
    pairs = [quantized_pair(rows, cols, 190 + 7 * i + rows // 16, use_dq) for i, rows in enumerate(rows_list)]
    x = synth.activations((3, cols), 199)
    ys = nf4.gemv_grouped([p[0] for p in pairs], dev_bf16(x))
    for (qw, p_ref, a_ref), y in zip(pairs, ys):
        check_matmul(y, oracle.matmul(p_ref, a_ref, qw.rows, cols, x), f"grouped {rows_list} {qw.rows}")
    nf4.check_device_error()


# --------------------------------------------------------------------------- 4-bit matmul + low-rank adapter

def lora_maps(rows, cols, r, seed):
    """bf16 adapter maps: down ~N(0, 1/cols) (so T is O(1)), up ~N(0, 0.02)"""
    down = synth.f32_to_bf16_bits((synth.rng(seed).standard_normal((r, cols)) / np.sqrt(cols)).astype(np.float32))
    up = synth.f32_to_bf16_bits((synth.rng(seed + 1).standard_normal((rows, r)) * 0.02).astype(np.float32))
    return down, up


@pytest.mark.parametrize("m", [1, 16, 65, 256, 300])
def test_gemm_lora_small(m):
    rows, cols, r = 256, 512, 16
    qw, p_ref, a_ref = quantized_pair(rows, cols, 111 + m, True)
    x = synth.activations((m, cols), 112 + m)
    down, up = lora_maps(rows, cols, r, 113 + m)
    y = nf4.gemm_lora(qw, dev_bf16(x), dev_bf16(down), dev_bf16(up), 2.0)
    check_matmul(y, oracle.matmul_lora(p_ref, a_ref, rows, cols, x, down, up, r, 2.0), f"gemm_lora m{m}")


@pytest.mark.parametrize("r", [16, 32])
@pytest.mark.parametrize("use_dq", [False, True])
def test_gemm_lora_ranks(r, use_dq):
    rows, cols, m = 384, 1024, 200
    qw, p_ref, a_ref = quantized_pair(rows, cols, 120 + r, use_dq)
    x = synth.activations((m, cols), 121 + r)
    down, up = lora_maps(rows, cols, r, 122 + r)
    y = nf4.gemm_lora(qw, dev_bf16(x), dev_bf16(down), dev_bf16(up), 32.0 / r)
    check_matmul(y, oracle.matmul_lora(p_ref, a_ref, rows, cols, x, down, up, r, 32.0 / r), f"gemm_lora r{r}")


@pytest.mark.parametrize("m", [65, 256, 300])
def test_gemm_lora_split(m):
    """few output tiles: the adapter stage rides with split 0 of each tile"""
    rows, cols, r = 256, 2048, 16
    qw, p_ref, a_ref = quantized_pair(rows, cols, 130 + m, True)
    x = synth.activations((m, cols), 131 + m)
    down, up = lora_maps(rows, cols, r, 132 + m)
    y = nf4.gemm_lora(qw, dev_bf16(x), dev_bf16(down), dev_bf16(up), 2.0)
    check_matmul(y, oracle.matmul_lora(p_ref, a_ref, rows, cols, x, down, up, r, 2.0), f"gemm_lora split m{m}")


def test_gemm_lora_zero_up_is_gemm_bit_exact_and_down_map():
    """with up = 0 the adapter stage adds exact zeros: the same bits as nf4_gemm (same tiles and splits).  The
    down map left in the workspace as a bf16 pair [hi | lo | 0] holds v = s * X . A^T: lo is at most half a bf16
    ulp of hi, and hi + lo is within 2^-15 relative of the oracle's fp64 value, plus fp32 summation error (1e-6 of
    sum |x a|)"""
    rows, cols, m, r = 4096, 4096, 256, 16
    qw, p_ref, a_ref = quantized_pair(rows, cols, 140, True)
    x = synth.activations((m, cols), 141)
    down, _ = lora_maps(rows, cols, r, 142)
    ws = torch.zeros(nf4.gemm_lora_workspace_bytes(qw, m), dtype=torch.uint8, device="cuda")
    y = nf4.gemm_lora(qw, dev_bf16(x), dev_bf16(down), torch.zeros(rows, r, dtype=torch.bfloat16, device="cuda"),
                      2.0, workspace=ws)
    assert torch.equal(y.view(torch.int16), nf4.gemm(qw, dev_bf16(x)).view(torch.int16))
    t = ws[:m * 64 * 2].view(torch.int16).view(m, 64).cpu().numpy().view(np.uint16)
    assert np.all(t[:, 2 * r:] == 0)
    hi = synth.bf16_bits_to_f32(t[:, :r]).astype(np.float64)
    lo = synth.bf16_bits_to_f32(t[:, r:2 * r]).astype(np.float64)
    v = hi + lo
    assert np.all(np.abs(lo) <= 2.0 ** -8 * np.abs(hi))  # lo is the rounding remainder of hi
    t_ref = oracle.lora_down(x, cols, down, r, 2.0)
    absdot = np.abs(synth.bf16_bits_to_f32(x).astype(np.float64)) @ np.abs(
        synth.bf16_bits_to_f32(down).astype(np.float64)).T
    assert np.all(np.abs(v - t_ref) <= 2.0 ** -15 * np.abs(t_ref) + 1e-6 * 2.0 * absdot)


def test_gemm_lora_adapter_only():
    """zero-code weight: Y is the adapter term alone"""
    rows, cols, m, r = 256, 1024, 300, 16
    p = torch.full((rows * cols // 2,), 0x77, dtype=torch.uint8, device="cuda")
    absmax = torch.ones(rows * cols // 64, dtype=torch.float32, device="cuda")
    qw = nf4.QuantizedWeight(packed=p, rows=rows, cols=cols, absmax=absmax)
    x = synth.activations((m, cols), 150)
    down, up = lora_maps(rows, cols, r, 151)
    y = nf4.gemm_lora(qw, dev_bf16(x), dev_bf16(down), dev_bf16(up), 2.0)
    ref = oracle.matmul_lora(np.full(rows * cols // 2, 0x77, np.uint8), np.ones(rows * cols // 64, np.float32),
                             rows, cols, x, down, up, r, 2.0)
    check_matmul(y, ref, "gemm_lora adapter only")


@pytest.mark.parametrize("m", [16, 256, 1024, 4096])
def test_gemm_lora_14336x4096_sampled(m):
    """W 14336x4096 NF4+DQ with an r = 16, alpha = 32 adapter at the prefill sizes: 2048 sampled outputs and
    all of row 0 against the oracle; ten identical calls give identical bits"""
    rows, cols, r = 14336, 4096, 16
    qw, p_ref, a_ref = quantized_pair(rows, cols, 1020, True)
    x = synth.activations((m, cols), 1021 + m)
    down, up = lora_maps(rows, cols, r, 160)
    ws = torch.zeros(nf4.gemm_lora_workspace_bytes(qw, m), dtype=torch.uint8, device="cuda")
    args = (qw, dev_bf16(x), dev_bf16(down), dev_bf16(up), 2.0)
    y = nf4.gemm_lora(*args, workspace=ws)
    for _ in range(3):
        assert torch.equal(nf4.gemm_lora(*args, workspace=ws).view(torch.int16), y.view(torch.int16))
    rg = synth.rng(170 + m)
    bs, ns = rg.integers(0, m, 2048), rg.integers(0, rows, 2048)
    ref = oracle.matmul_lora_sampled(p_ref, a_ref, rows, cols, x, down, up, r, 2.0, bs, ns)
    full_row = oracle.matmul_lora(p_ref, a_ref, rows, cols, x[:1], down, up, r, 2.0)
    rms = np.sqrt(np.mean(full_row ** 2))
    got = y.float().cpu().numpy().astype(np.float64)[bs, ns]
    assert np.all(np.abs(got - ref) <= REL_TOL * np.maximum(np.abs(ref), FLOOR * rms))
    check_matmul(y[:1], full_row, f"gemm_lora m{m} row 0")
    nf4.check_device_error()


# --------------------------------------------------------------------------- input gradient dX = dY . Wc

def check_dx_sampled(dx: torch.Tensor, p_ref, a_ref, rows, cols, dy, seed, count=2048):
    """`count` sampled outputs against the oracle (rms floor from the first full row), plus row 0 in full"""
    m = dy.shape[0]
    r = synth.rng(seed)
    bs, ks = r.integers(0, m, count), r.integers(0, cols, count)
    ref = oracle.matmul_dx_sampled(p_ref, a_ref, rows, cols, dy, bs, ks)
    full_row = oracle.matmul_dx(p_ref, a_ref, rows, cols, dy[:1])
    rms = np.sqrt(np.mean(full_row ** 2))
    got = dx.float().cpu().numpy().astype(np.float64)[bs, ks]
    bad = np.abs(got - ref) > REL_TOL * np.maximum(np.abs(ref), FLOOR * rms)
    assert not bad.any(), f"{bad.sum()} of {count} sampled dx outputs beyond tolerance"
    check_matmul(dx[:1], full_row, "dx row 0")


@pytest.mark.parametrize("m", [1, 16, 100, 256, 300])
def test_gemm_dx_small(m):
    rows, cols = 256, 512
    qw, p_ref, a_ref = quantized_pair(rows, cols, 81 + m, True)
    dy = synth.activations((m, rows), 82 + m)
    dx = nf4.gemm_dx(qw, dev_bf16(dy))
    assert dx.shape == (m, cols)
    check_matmul(dx, oracle.matmul_dx(p_ref, a_ref, rows, cols, dy), f"gemm_dx m{m}")


def test_gemm_dx_one_hot_rows_bit_exact():
    """one-hot gradient rows read weight rows back: dX = bf16_rn(code * a^) of that row, bit for bit
    (a single nonzero product per output, so the fp32 sum and the bf16 rounding are exact); covers
    weight rows in every 16-row MMA step and 8-row swizzle group of a stage, and both column halves"""
    rows, cols = 192, 384
    qw, p_ref, a_ref = quantized_pair(rows, cols, 5, True)
    wc = oracle.dequantize(p_ref, a_ref, rows * cols, 64, "bf16").reshape(rows, cols)
    ns = [0, 1, 7, 8, 15, 16, 31, 47, 63, 64, 100, 127, 128, 150, 190, 191]
    dy = synth.f32_to_bf16_bits(np.eye(rows, dtype=np.float32)[ns])
    dx = nf4.gemm_dx(qw, dev_bf16(dy))
    assert np.array_equal(host_bf16_bits(dx), wc[ns])


@pytest.mark.parametrize("cols", [384, 1024, 4096])
@pytest.mark.parametrize("use_dq,code", [(False, "e4m3"), (True, "e4m3"), (True, "int8")])
def test_gemm_dx_scale_paths(cols, use_dq, code):
    """plain fp32 and double-quantized scales; scale rows that are (1024, 4096) and are not (384) whole
    16-byte units (TMA chunks vs per-block loads)"""
    rows, m = 128, 160
    qw, p_ref, a_ref = quantized_pair(rows, cols, 91 + cols, use_dq, code)
    dy = synth.activations((m, rows), 92 + cols)
    dx = nf4.gemm_dx(qw, dev_bf16(dy))
    check_matmul(dx, oracle.matmul_dx(p_ref, a_ref, rows, cols, dy), f"gemm_dx cols{cols} dq{use_dq} {code}")


@pytest.mark.parametrize("m", [65, 256, 300])
def test_gemm_dx_split_k(m):
    """few output tiles: the reduction over weight rows is split across CTAs"""
    rows, cols = 2048, 256
    qw, p_ref, a_ref = quantized_pair(rows, cols, 95 + m, True)
    assert nf4.gemm_dx_workspace_bytes(qw, m) > 0
    dy = synth.activations((m, rows), 96 + m)
    dx = nf4.gemm_dx(qw, dev_bf16(dy))
    check_matmul(dx, oracle.matmul_dx(p_ref, a_ref, rows, cols, dy), f"gemm_dx split m{m}")


@pytest.mark.parametrize("shape", [(14336, 4096), (4096, 14336), (4096, 4096)])
@pytest.mark.parametrize("m", [256, 1024, 4096])
def test_gemm_dx_llama_shapes_sampled(shape, m):
    """dX for the 8B-shaped projections (gate/up 14336x4096, down 4096x14336, 4096^2) at the prefill
    token counts: 2048 sampled outputs and all of row 0 against the oracle"""
    rows, cols = shape
    qw, p_ref, a_ref = quantized_pair(rows, cols, 1030 + rows // 1024, True)
    dy = synth.activations((m, rows), 1031 + m)
    dx = nf4.gemm_dx(qw, dev_bf16(dy))
    check_dx_sampled(dx, p_ref, a_ref, rows, cols, dy, 11 + m)
    nf4.check_device_error()


@pytest.mark.parametrize("rows,cols,m", [(14336, 4096, 1024), (4096, 4096, 256), (4096, 14336, 4096)])
def test_gemm_dx_repeatable(rows, cols, m):
    """ten identical calls (persistent CTAs cycling their rings, both accumulators; split path at m=256)
    give identical bits"""
    w = synth.normal_weights((rows, cols), 2030)
    qw = nf4.quantize_weight(dev(w))
    dy = dev_bf16(synth.activations((m, rows), 2031))
    ws = torch.zeros(max(nf4.gemm_dx_workspace_bytes(qw, m), 16), dtype=torch.uint8, device="cuda")
    ref = nf4.gemm_dx(qw, dy, workspace=ws).view(torch.int16).clone()
    for _ in range(10):
        assert torch.equal(nf4.gemm_dx(qw, dy, workspace=ws).view(torch.int16), ref)
    nf4.check_device_error()


def test_gemm_dx_adjoint_of_gemm():
    """<dY, X . Wc^T> = <dY . Wc, X> between the library's own forward and gradient products at a full
    prefill size (only bf16 output rounding separates the two sides)"""
    rows, cols, m = 4096, 4096, 512
    w = synth.normal_weights((rows, cols), 2040)
    qw = nf4.quantize_weight(dev(w))
    x = dev_bf16(synth.activations((m, cols), 2041))
    dy = dev_bf16(synth.activations((m, rows), 2042))
    t1 = dy.double() * nf4.gemm(qw, x).double()
    t2 = nf4.gemm_dx(qw, dy).double() * x.double()
    # each output carries at most half a bf16 ulp (2^-9 relative) of independent rounding: the sums differ
    # by a random walk of those, bounded here at 8 standard deviations
    scale = float(torch.sqrt((t1 ** 2).sum() + (t2 ** 2).sum()))
    assert abs(float(t1.sum()) - float(t2.sum())) <= 2.0 ** -6 * scale


# --------------------------------------------------------------------------- whole 8B-shaped model

def test_whole_model_8b():
    """An 8B-shaped decoder stack: 32 layers x (q, k, v, o, gate, up, down), 6.98e9 bf16 weights ~N(0, 0.02), each
    matrix from its own seed, quantized to NF4 with E4M3 double quant on the GPU, then a GEMV pass over all 224
    matrices in layer order at batch 1, 4 and 8.  One matrix of each projection type (from different layers) is
    checked in full against the oracle: packed codes, 8-bit absmax codes, second-level scales and mean bit for bit,
    and 512 sampled outputs of every batch within the matmul tolerance.  Storage matches the 4.127 bits/param
    figure (3.60 GB for the stack)."""
    torch.cuda.empty_cache()
    shapes = synth.LLAMA8B_LAYER
    checked = {(3 + 5 * p) % synth.LLAMA8B_LAYERS: p for p in range(len(shapes))}  # layer -> projection
    records, sources, total_params, stored = [], {}, 0, 0
    for layer in range(synth.LLAMA8B_LAYERS):
        for p, (name, rows, cols) in enumerate(shapes):
            w = synth.normal_weights_device((rows, cols), synth.layer_seed(layer, p))
            qw = nf4.quantize_weight(w, use_double_quant=True, code="e4m3")
            if checked.get(layer) == p:
                sources[(layer, p)] = w.view(torch.int16).cpu().numpy().view(np.uint16)
            del w
            records.append((layer, p, qw))
            total_params += rows * cols
            stored += qw.storage_bytes()
    assert total_params == 6_979_321_856
    assert abs(stored * 8 / total_params - (4 + 8 / 64 + 32 / (64 * 256))) < 1e-3
    xs = {b: (synth.activations_device((b, 4096), 3000 + b), synth.activations_device((b, 14336), 3100 + b))
          for b in (1, 4, 8)}
    outs = {}
    for b, (x_model, x_ffn) in xs.items():  # one pass over the stack, layer order
        for layer, p, qw in records:
            y = nf4.gemv(qw, x_ffn if shapes[p][0] == "down" else x_model)
            if (layer, p) in sources:
                outs[(layer, p, b)] = y
    nf4.check_device_error()
    r = synth.rng(77)
    for (layer, p), src in sources.items():
        name, rows, cols = shapes[p]
        qw = records[layer * len(shapes) + p][2]
        w32 = synth.bf16_bits_to_f32(src.reshape(-1))
        p_ref, a_ref = oracle.quantize(w32)
        q_ref, s_ref, m_ref = oracle.double_quant(a_ref, 256, oracle.DQ_E4M3)
        assert np.array_equal(qw.packed.cpu().numpy(), p_ref), (layer, name)
        assert np.array_equal(qw.absmax_q.cpu().numpy(), q_ref), (layer, name)
        assert np.array_equal(qw.absmax_scale.cpu().numpy().view(np.uint32), s_ref.view(np.uint32)), (layer, name)
        assert np.float32(qw.absmax_mean.item()).view(np.uint32) == np.float32(m_ref).view(np.uint32)
        a_hat = oracle.absmax_reconstruct(q_ref, s_ref, m_ref, 256, oracle.DQ_E4M3)
        for b, (x_model, x_ffn) in xs.items():
            x = (x_ffn if name == "down" else x_model).view(torch.int16).cpu().numpy().view(np.uint16)
            bs, ns = r.integers(0, b, 512), r.integers(0, rows, 512)
            ref = oracle.matmul_sampled(p_ref, a_hat, rows, cols, x, bs, ns)
            full_row = oracle.matmul(p_ref, a_hat, rows, cols, x[:1])
            rms = np.sqrt(np.mean(full_row ** 2))
            got = outs[(layer, p, b)].float().cpu().numpy().astype(np.float64)[bs, ns]
            bad = np.abs(got - ref) > REL_TOL * np.maximum(np.abs(ref), FLOOR * rms)
            assert not bad.any(), (layer, name, b, int(bad.sum()))
    del records, outs
    torch.cuda.empty_cache()


# --------------------------------------------------------------------------- failure path

def test_bounded_wait_times_out_and_context_survives():
    """A device-side wait that nothing completes gives up after the library's bound, reports NF4_ERR_TIMEOUT
    through nf4_check_device_error, and leaves the context usable (a quantization afterwards is exact)."""
    from qlora_block_absmax_b200 import _lib
    lib = _lib.load()
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.nf4_selftest_wait_timeout(stream) == 0
    with pytest.raises(_lib.NF4Error) as e:
        nf4.check_device_error()
    assert "TIMEOUT" in str(e.value)
    nf4.check_device_error()  # the word was cleared
    w = synth.normal_weights((4096,), 5)
    p_ref, a_ref = oracle.quantize(w)
    p, a = nf4.quantize(dev(w))
    assert np.array_equal(p.cpu().numpy(), p_ref)
    assert np.array_equal(a.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))
    nf4.check_device_error()

