"""Pins of the CPU oracle to facts fixed outside itself: library routines
(statistics.NormalDist, math.fsum, torch casts, numpy searchsorted), closed
forms, the pages' worked example and storage figures, invariants the pages
state, and brute force on tiny inputs.  CPU only."""
import math
import statistics
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from qlora_block_absmax_b200 import synth
from tests.conftest import read_golden

PSTAR = 0.5 * ((1 - 1 / 30) + (1 - 1 / 32))


def f32(x):
    return struct.unpack("<f", struct.pack("<f", x))[0]


# ---------------------------------------------------------------- code book

def test_codebook_matches_independent_quantile_routine():
    """Same definition evaluated with statistics.NormalDist.inv_cdf (a
    different inverse-CDF algorithm) agrees bit for bit in fp32."""
    _, c32 = oracle.codebook()
    nd = statistics.NormalDist()
    neg = [-nd.inv_cdf(0.5 + (PSTAR - 0.5) * (k / 7)) for k in range(7, 0, -1)]
    pos = [nd.inv_cdf(0.5 + (PSTAR - 0.5) * (k / 8)) for k in range(1, 9)]
    v = np.array(neg + [0.0] + pos)
    v = v / np.abs(v).max()
    assert np.array_equal(v.astype(np.float32), c32)


def test_codebook_equal_share_of_bell_curve():
    """'How NF4 works': each level covers an equal share of the normal curve --
    mapping the levels back through the normal CDF gives equally spaced
    probabilities (8 steps above zero, 7 below)."""
    c64, _ = oracle.codebook()
    zmax = statistics.NormalDist().inv_cdf(PSTAR)
    cdf = [0.5 * (1 + math.erf(c * zmax / math.sqrt(2))) for c in c64]
    pos = np.diff(cdf[7:])
    neg = np.diff(cdf[:8])
    assert np.allclose(pos, (PSTAR - 0.5) / 8, rtol=0, atol=1e-12)
    assert np.allclose(neg, (PSTAR - 0.5) / 7, rtol=0, atol=1e-12)


def test_codebook_shape():
    c64, c32 = oracle.codebook()
    assert c32[0] == -1.0 and c32[15] == 1.0
    assert struct.pack("<f", c32[7]) == b"\x00\x00\x00\x00"  # exact +0
    assert np.all(np.diff(c32) > 0)
    assert (c32 < 0).sum() == 7 and (c32 > 0).sum() == 8
    # finer marks near zero, coarser far out ('How NF4 works')
    gaps_pos = np.diff(c64[7:])
    gaps_neg = np.diff(c64[:8])[::-1]        # from zero outward
    assert np.all(np.diff(gaps_pos) > 0) and np.all(np.diff(gaps_neg) > 0)


# ---------------------------------------------------------------- bf16

def test_bf16_rounding_matches_torch_cast():
    r = synth.rng(7)
    x = np.concatenate([
        r.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        (r.standard_normal(2000) * 1e30).astype(np.float32),
        np.array([0.0, -0.0, 1.0, 3.0e38, -3.0e38, 1e-40, -1e-40], np.float32),
    ])
    # exact ties: bf16 value plus half an ulp
    ties = (synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x[:500])).view(np.uint32) | 0x8000).view(np.float32)
    x = np.concatenate([x, ties])
    want = synth.f32_to_bf16_bits(x)
    got = np.array([oracle.bf16_rn(float(v)) for v in x], np.uint16)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------- nearest code

def _midpoints():
    _, c32 = oracle.codebook()
    return np.array([(float(c32[i]) + float(c32[i + 1])) / 2 for i in range(15)])  # exact in fp64


def test_nearest_code_equals_midpoint_count_near_every_midpoint():
    """argmin-distance (the oracle) == number of exact midpoints strictly below
    x (numpy searchsorted), exhaustively for the 2x64 fp32 values around every
    midpoint and for random values in [-1, 1]."""
    mids = _midpoints()
    xs = []
    for m in mids:
        b = np.array([m], np.float32).view(np.int32)[0]
        for d in range(-64, 65):
            xs.append(np.array([b + d], np.int32).view(np.float32)[0])
    xs = np.concatenate([np.array(xs, np.float32),
                         synth.rng(11).uniform(-1, 1, 20000).astype(np.float32),
                         np.array([-1, 1, 0, -0.0], np.float32)])
    want = np.searchsorted(mids, xs.astype(np.float64), side="left")
    got = np.array([oracle.nearest_code(float(x)) for x in xs])
    assert np.array_equal(got, want)


def test_nearest_code_special_values():
    _, c32 = oracle.codebook()
    for i, c in enumerate(c32):
        assert oracle.nearest_code(float(c)) == i
    assert oracle.nearest_code(0.0) == 7 and oracle.nearest_code(-0.0) == 7
    assert oracle.nearest_code(1.0) == 15 and oracle.nearest_code(-1.0) == 0


# ---------------------------------------------------------------- level-1 quantize

def _brute_quantize(w, bs):
    """numpy brute force: fp32 division by the block absmax, argmin |x - c|."""
    _, c32 = oracle.codebook()
    n = w.size
    codes = np.zeros(n, np.uint8)
    absmax = np.zeros((n + bs - 1) // bs, np.float32)
    for b in range(absmax.size):
        blk = w[b * bs:(b + 1) * bs]
        a = np.abs(blk).max()
        absmax[b] = a
        if a == 0:
            codes[b * bs:b * bs + blk.size] = 7
            continue
        x = (blk / a).astype(np.float32)
        d = np.abs(x.astype(np.float64)[:, None] - c32.astype(np.float64)[None, :])
        codes[b * bs:b * bs + blk.size] = np.argmin(d, axis=1)  # first minimum = lower index
    if n % 2:
        codes = np.append(codes, 7)
    packed = (codes[0::2] << 4) | codes[1::2]
    return packed.astype(np.uint8), absmax


@pytest.mark.parametrize("n,bs", [(1, 64), (63, 64), (64, 64), (65, 64), (127, 64), (4097, 64), (1000, 32)])
def test_quantize_brute_force_tiny(n, bs):
    w = synth.normal_weights((n,), 100 + n)
    w[::17] = 0.0
    p, a = oracle.quantize(w, bs)
    bp, ba = _brute_quantize(w, bs)
    assert np.array_equal(a, ba)
    assert np.array_equal(p, bp)


def test_quantize_packing_order_hand_example():
    """Step 4: two codes per byte; first element in the high nibble; odd tail
    padded with the zero code."""
    w = np.array([1.0, -1.0, 0.0, 0.5, 0.25], np.float32)
    p, a = oracle.quantize(w, 64)
    # 0.5 lies between c12 = 0.4407 and c13 = 0.5626, nearer c12; 0.25 nearest c10 = 0.2461
    assert a.tolist() == [1.0]
    assert p.tolist() == [0xF0, 0x7C, 0xA7]


def test_quantize_invariants():
    w = synth.normal_weights((64 * 500,), 5)
    w[64 * 3:64 * 4] = 0.0              # all-zero block
    w[64 * 7 + 5] = -0.0
    p, a = oracle.quantize(w, 64)
    codes = np.empty(w.size, np.uint8)
    codes[0::2] = p >> 4
    codes[1::2] = p & 15
    blocks = w.reshape(-1, 64)
    cb = codes.reshape(-1, 64)
    assert np.array_equal(a, np.abs(blocks).max(axis=1))
    for b in range(blocks.shape[0]):
        if a[b] == 0:
            assert np.all(cb[b] == 7)
            continue
        j = np.argmax(np.abs(blocks[b]))
        assert cb[b, j] == (15 if blocks[b, j] > 0 else 0)   # max element -> +-1 code
    assert np.all(codes[w == 0] == 7)                          # zeros -> zero code


def test_quantize_dequantize_roundtrip_is_identity_on_codes():
    w = synth.normal_weights((64 * 2000 + 31,), 9)
    p, a = oracle.quantize(w, 64)
    wh = oracle.dequantize(p, a, w.size, 64)
    p2, a2 = oracle.quantize(wh, 64)
    assert np.array_equal(p2, p) and np.array_equal(a2, a)


def test_quantize_bf16_path_is_exact_widening():
    wb = synth.normal_weights((64 * 100 + 3,), 21, dtype="bf16")
    p1, a1 = oracle.quantize(wb, 64)
    p2, a2 = oracle.quantize(synth.bf16_bits_to_f32(wb), 64)
    assert np.array_equal(p1, p2) and np.array_equal(a1, a2)


# ---------------------------------------------------------------- exact sum

def test_exact_sum_matches_fsum():
    r = synth.rng(3)
    cases = [
        np.abs(r.standard_normal(10000)).astype(np.float32) * np.float32(0.05),
        (r.standard_normal(5000) * np.exp(r.uniform(-60, 60, 5000))).astype(np.float32),
        np.array([1e30, 1.0, -1e30, 1e-30], np.float32),
        np.array([3.0e38, 3.0e38, -3.0e38], np.float32),
        np.array([1e-45, 2e-45, -1e-45, 1e-40], np.float32),
        np.array([2.0 ** 60, 1.0, 2.0 ** -60], np.float32),
        np.zeros(7, np.float32),
    ]
    for a in cases:
        assert oracle.exact_sum(a) == math.fsum(a.astype(np.float64).tolist())


# ---------------------------------------------------------------- E4M3

def test_e4m3_decode_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    ref = codes.to(torch.float32).numpy()
    got = np.array([oracle.e4m3_decode(c) for c in range(256)], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2
    assert np.array_equal(got[~nan], ref[~nan])
    assert got[0x7e] == 448.0 and len(set(got[~nan].tolist())) == 253


def test_e4m3_encode_matches_torch_rne_inside_range():
    vals = np.array(sorted(set(oracle.e4m3_decode(c) for c in range(0x7f))), np.float64)
    mids = (vals[:-1] + vals[1:]) / 2                       # exact ties
    r = synth.rng(4)
    ys = np.concatenate([vals, -vals, mids, -mids,
                         r.uniform(-448, 448, 5000), r.standard_normal(3000) * 0.01,
                         np.nextafter(mids, 0), np.nextafter(mids, 1000)]).astype(np.float32)
    ys = ys[np.abs(ys) <= 448]
    ref = torch.from_numpy(ys).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(y)) for y in ys], np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_encode_saturates():
    for y in [448.0, 449.0, 464.0, 1e6, 3e38]:
        assert oracle.e4m3_encode(y) == 0x7e and oracle.e4m3_encode(-y) == 0xfe


# ---------------------------------------------------------------- second level / worked example

def test_worked_example_int8():
    g = read_golden("worked_example_int8.txt")
    w = np.array(g["weights"], np.float32)
    q, scale = oracle.blockwise_8bit(w, 256, oracle.DQ_INT8)
    assert scale[0] == np.float32(g["absmax"][0])
    assert np.array_equal(q.view(np.int8).astype(int), np.array(g["codes"], int))
    assert np.allclose(w / scale[0], g["scaled"], atol=1e-7)
    for code, approx in zip(g["dequant_of"], g["dequant_approx"]):
        v = oracle.blockwise_8bit_value(int(np.int8(code).view(np.uint8)), float(scale[0]), oracle.DQ_INT8)
        assert abs(v - approx) < 1e-4
    errs = [abs(oracle.blockwise_8bit_value(int(qq), float(scale[0]), oracle.DQ_INT8) - float(ww))
            for qq, ww in zip(q[:2], w[:2])]
    assert np.allclose(errs, g["error_approx"], atol=5e-4)


@pytest.mark.parametrize("code,top", [(oracle.DQ_E4M3, 0x7e), (oracle.DQ_INT8, 127)])
def test_blockwise_8bit_block_max_maps_to_top_code(code, top):
    v = synth.rng(8).standard_normal(256 * 9 + 77).astype(np.float32)
    q, scale = oracle.blockwise_8bit(v, 256, code)
    for g in range(scale.size):
        blk = v[g * 256:(g + 1) * 256]
        j = np.argmax(np.abs(blk))
        assert scale[g] == np.abs(blk).max()
        want = top if blk[j] > 0 else (top | 0x80 if code == oracle.DQ_E4M3 else (256 - top))
        assert q[g * 256 + j] == want
        assert oracle.blockwise_8bit_value(int(q[g * 256 + j]), float(scale[g]), code) == blk[j]


def test_double_quant_mean_and_reconstruction_bound():
    w = synth.add_outliers(synth.normal_weights((64 * 4096,), 31), 32)
    _, a = oracle.quantize(w, 64)
    for code, rel in [(oracle.DQ_E4M3, 2.0 ** -4), (oracle.DQ_INT8, 1.0 / 254)]:
        q, scale, mean = oracle.double_quant(a, 256, code)
        exact = sum(Fraction(float(x)) for x in a) / a.size          # exact mean
        assert mean == f32(float(Fraction(math.fsum(a.astype(np.float64))) / a.size))
        assert abs(Fraction(mean) - exact) <= abs(exact) * Fraction(2) ** -24
        ah = oracle.absmax_reconstruct(q, scale, mean, 256, code)
        for g in range(scale.size):
            blk = slice(g * 256, (g + 1) * 256)
            # 8-bit grid error: half a step of the code around the block absmax of residuals
            assert np.all(np.abs(ah[blk] - a[blk]) <= scale[g] * rel * 1.0001 + 1e-7)


def test_double_quant_degenerate_constant_absmax():
    a = np.full(1000, 0.375, np.float32)
    q, scale, mean = oracle.double_quant(a, 256, oracle.DQ_E4M3)
    assert mean == 0.375 and np.all(scale == 0) and np.all(q == 0)
    assert np.all(oracle.absmax_reconstruct(q, scale, mean) == a)


# ---------------------------------------------------------------- storage arithmetic

def storage_bytes(n, bs=64, dq=True, dq_bs=256):
    nb = -(-n // bs)
    if not dq:
        return -(-n // 2) + 4 * nb
    return -(-n // 2) + nb + 4 * (-(-nb // dq_bs)) + 4


def test_storage_matches_pages_figures():
    g = read_golden("storage_claims.txt")
    n = 4096 * 4096
    bits = 8 * storage_bytes(n) / n
    assert abs(bits - (4 + 8 / 64 + 32 / (64 * 256) + 32 / n)) < 1e-9   # ~4.127 (+ one fp32 mean)
    saving = 8 * (storage_bytes(n, dq=False) - storage_bytes(n)) / n
    assert abs(saving - g["dq_saving_bits_per_param"][0]) < 0.05        # "about 0.4"
    params = synth.LLAMA8B_LAYERS * sum(r * c for _, r, c in synth.LLAMA8B_LAYER)
    total = synth.LLAMA8B_LAYERS * sum(storage_bytes(r * c) for _, r, c in synth.LLAMA8B_LAYER)
    gb = total / 1e9
    assert g["int4_7b_gb_before_scales"][0] < gb < g["nf4_7b_gb"][0]   # 3.5 GB + small overhead, < ~4 GB
    assert abs(params * 2 / 1e9 - g["fp16_7b_gb"][0]) < 0.2 * g["fp16_7b_gb"][0]


# ---------------------------------------------------------------- dequantize

def test_dequantize_against_numpy_products():
    w = synth.normal_weights((64 * 300 + 5,), 41)
    p, a = oracle.quantize(w, 64)
    _, c32 = oracle.codebook()
    codes = np.empty(p.size * 2, np.uint8)
    codes[0::2] = p >> 4
    codes[1::2] = p & 15
    codes = codes[:w.size]
    want = (c32[codes] * np.repeat(a, 64)[:w.size]).astype(np.float32)
    got = oracle.dequantize(p, a, w.size, 64)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    got16 = oracle.dequantize(p, a, w.size, 64, "bf16")
    assert np.array_equal(got16, synth.f32_to_bf16_bits(want))
    # block max reconstructs to +-absmax exactly; zero codes give 0
    blocks = w[:64 * 300].reshape(-1, 64)
    j = np.argmax(np.abs(blocks), axis=1)
    assert np.array_equal(np.abs(got[:64 * 300].reshape(-1, 64)[np.arange(300), j]), a[:300])
    assert np.all(got[codes == 7] == 0)


# ---------------------------------------------------------------- matmul

def test_matmul_one_hot_columns_and_numpy_dot():
    N, K = 48, 192
    w = synth.normal_weights((N, K), 51)
    p, a = oracle.quantize(w, 64)
    wc = synth.bf16_bits_to_f32(oracle.dequantize(p, a, N * K, 64, "bf16")).reshape(N, K)
    # one-hot activations pick columns of the 16-bit expanded weight exactly
    eye = synth.f32_to_bf16_bits(np.eye(K, dtype=np.float32)[[0, 5, 63, 64, 191]])
    y = oracle.matmul(p, a, N, K, eye)
    assert np.array_equal(y, wc[:, [0, 5, 63, 64, 191]].T.astype(np.float64))
    x = synth.activations((3, K), 52)
    y = oracle.matmul(p, a, N, K, x)
    ref = synth.bf16_bits_to_f32(x).astype(np.float64) @ wc.astype(np.float64).T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-15)
    ys = oracle.matmul_sampled(p, a, N, K, x, np.array([0, 2, 1]), np.array([0, 47, 13]))
    assert np.array_equal(ys, y[[0, 2, 1], [0, 47, 13]])


def test_matmul_zero_codes_give_zero():
    N, K = 16, 128
    p = np.full(N * K // 2, 0x77, np.uint8)
    a = np.ones(N * K // 64, np.float32)
    x = synth.activations((2, K), 3)
    assert np.all(oracle.matmul(p, a, N, K, x) == 0)



# ---------------------------------------------------------------- input gradient (dx = dy . Wc)

def test_matmul_dx_one_hot_rows_are_weight_rows():
    """dy = e_n picks row n of the 16-bit expanded weight, exactly (catches a
    transposed operand or a wrong row index)."""
    N, K = 80, 192
    w = synth.normal_weights((N, K), 61)
    p, a = oracle.quantize(w, 64)
    wc = synth.bf16_bits_to_f32(oracle.dequantize(p, a, N * K, 64, "bf16")).reshape(N, K)
    rows = [0, 1, 63, 64, 79]
    eye = synth.f32_to_bf16_bits(np.eye(N, dtype=np.float32)[rows])
    dx = oracle.matmul_dx(p, a, N, K, eye)
    assert np.array_equal(dx, wc[rows].astype(np.float64))


def test_matmul_dx_adjoint_of_forward():
    """<dy, x . Wc^T> = <dy . Wc, x> for every x, dy: the gradient is the
    adjoint of the forward map (pinned on its own), on a non-square weight so a
    transposed weight cannot pass."""
    N, K = 128, 320
    w = synth.normal_weights((N, K), 62)
    p, a = oracle.quantize(w, 64)
    x = synth.activations((5, K), 63)
    dy = synth.activations((5, N), 64)
    y = oracle.matmul(p, a, N, K, x)
    dx = oracle.matmul_dx(p, a, N, K, dy)
    lhs = np.sum(synth.bf16_bits_to_f32(dy).astype(np.float64) * y)
    rhs = np.sum(dx * synth.bf16_bits_to_f32(x).astype(np.float64))
    assert abs(lhs - rhs) <= 1e-12 * max(abs(lhs), 1.0)
    # the same identity fails for the transpose-free mistake dx = dy . Wc[:, reversed k]
    assert abs(lhs - np.sum(dx[:, ::-1] * synth.bf16_bits_to_f32(x).astype(np.float64))) > 1e-6


def test_matmul_dx_numpy_product_and_sampled():
    N, K = 96, 256
    w = synth.normal_weights((N, K), 65)
    p, a = oracle.quantize(w, 64)
    wc = synth.bf16_bits_to_f32(oracle.dequantize(p, a, N * K, 64, "bf16")).reshape(N, K)
    dy = synth.activations((4, N), 66)
    dx = oracle.matmul_dx(p, a, N, K, dy)
    ref = synth.bf16_bits_to_f32(dy).astype(np.float64) @ wc.astype(np.float64)
    assert np.allclose(dx, ref, rtol=1e-12, atol=1e-15)
    bs, ks = np.array([0, 3, 2, 1]), np.array([0, 255, 64, 129])
    assert np.array_equal(oracle.matmul_dx_sampled(p, a, N, K, dy, bs, ks), dx[bs, ks])


def test_matmul_dx_zero_codes_give_zero():
    N, K = 64, 128
    p = np.full(N * K // 2, 0x77, np.uint8)
    a = np.ones(N * K // 64, np.float32)
    assert np.all(oracle.matmul_dx(p, a, N, K, synth.activations((2, N), 4)) == 0)


# ---------------------------------------------------------------- low-rank adapter on the 4-bit matmul

def _bf16(a):
    return synth.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def test_lora_zero_adapter_is_the_plain_matmul():
    """an all-zero up map, or scale 0, leaves exactly the 4-bit product"""
    N, K, r = 64, 192, 16
    p, a = oracle.quantize(synth.normal_weights((N, K), 71), 64)
    x = synth.activations((3, K), 72)
    A = synth.activations((r, K), 73)
    B = synth.activations((N, r), 74)
    base = oracle.matmul(p, a, N, K, x)
    assert np.array_equal(oracle.matmul_lora(p, a, N, K, x, A, np.zeros((N, r), np.uint16), r, 2.0), base)
    assert np.array_equal(oracle.matmul_lora(p, a, N, K, x, A, B, r, 0.0), base)


def test_lora_one_hot_down_map_on_zero_weight():
    """zero-code weight (Wc = 0) and one-hot down-map rows A[j] = e_{k_j}: t = s * x[:, k_j] and y = t . B^T,
    checked against a numpy product"""
    N, K, r = 48, 128, 16
    p = np.full(N * K // 2, 0x77, np.uint8)
    a = np.ones(N * K // 64, np.float32)
    ks = np.array([0, 1, 5, 63, 64, 65, 100, 127, 2, 3, 4, 6, 7, 8, 9, 10])
    A = _bf16(np.eye(K, dtype=np.float32)[ks])
    x = synth.activations((5, K), 75)
    B = synth.activations((N, r), 76)
    t = oracle.lora_down(x, K, A, r, 2.0)
    xf = synth.bf16_bits_to_f32(x)
    assert np.array_equal(t, 2.0 * xf[:, ks].astype(np.float64))
    y = oracle.matmul_lora(p, a, N, K, x, A, B, r, 2.0)
    ref = (2.0 * xf[:, ks]).astype(np.float64) @ synth.bf16_bits_to_f32(B).astype(np.float64).T
    assert np.allclose(y, ref, rtol=1e-13, atol=1e-13)


def test_lora_down_matches_numpy():
    """t = s * x . A^T against a numpy fp64 product, for two scales (the map is linear in s)"""
    K, r = 320, 16
    x = synth.activations((7, K), 77)
    A = synth.activations((r, K), 78)
    prod = synth.bf16_bits_to_f32(x).astype(np.float64) @ synth.bf16_bits_to_f32(A).astype(np.float64).T
    assert np.allclose(oracle.lora_down(x, K, A, r, 2.0), 2.0 * prod, rtol=1e-13, atol=1e-12)
    assert np.allclose(oracle.lora_down(x, K, A, r, 0.375), 0.375 * prod, rtol=1e-13, atol=1e-12)


def test_lora_sum_of_parts():
    """y = x . Wc^T + t . B^T term by term: the adapter part equals the zero-weight case"""
    N, K, r = 64, 256, 16
    p, a = oracle.quantize(synth.normal_weights((N, K), 79), 64)
    x = synth.activations((4, K), 80)
    A = synth.activations((r, K), 81)
    B = synth.activations((N, r), 82)
    y = oracle.matmul_lora(p, a, N, K, x, A, B, r, 2.0)
    zero = np.full(N * K // 2, 0x77, np.uint8)
    adapter = oracle.matmul_lora(zero, a, N, K, x, A, B, r, 2.0)
    assert np.allclose(y, oracle.matmul(p, a, N, K, x) + adapter, rtol=1e-13, atol=1e-12)
    bs, ns = np.array([0, 3, 2, 1, 3]), np.array([0, 63, 17, 40, 5])
    assert np.array_equal(oracle.matmul_lora_sampled(p, a, N, K, x, A, B, r, 2.0, bs, ns), y[bs, ns])


# ---------------------------------------------------------------- FP4 variant (E2M1 / 6, stored as the bit pattern)

# OCP microscaling spec, FP4 E2M1: the value of each 3-bit magnitude pattern e1 e0 m (bias 1, subnormals at e = 0)
E2M1_SPEC = {0b000: 0.0, 0b001: 0.5, 0b010: 1.0, 0b011: 1.5, 0b100: 2.0, 0b101: 3.0, 0b110: 4.0, 0b111: 6.0}


def test_fp4_codebook_is_the_e2m1_table_over_6():
    c64, c32 = oracle.fp4_codebook()
    for nib in range(16):
        v = E2M1_SPEC[nib & 7] / 6.0 * (-1.0 if nib & 8 else 1.0)
        assert c64[nib] == v and c32[nib] == np.float32(v)
        assert math.copysign(1.0, c64[nib]) == (-1.0 if nib & 8 else 1.0)  # pattern 8 is -0


def _fp4_brute(x: float) -> int:
    """exact nearest of the fp32 levels by rational arithmetic; tie -> even mantissa bit; sign of x kept"""
    _, c32 = oracle.fp4_codebook()
    ax = abs(Fraction(float(x)))
    best, bd = None, None
    for k in range(8):
        d = abs(ax - Fraction(float(c32[k])))
        if bd is None or d < bd or (d == bd and k % 2 == 0):
            best, bd = k, d
    return best | (8 if math.copysign(1.0, x) < 0 else 0)


def test_fp4_nearest_code_brute_force():
    _, c32 = oracle.fp4_codebook()
    xs = [0.0, -0.0, 1.0, -1.0, 1e-30, -1e-30]
    for k in range(8):  # every level, its neighbours in fp32, and every midpoint with its neighbours
        lv = np.float32(c32[k])
        xs += [float(lv), float(np.nextafter(lv, np.float32(2))), float(np.nextafter(lv, np.float32(-2)))]
        if k < 7:
            mid = (Fraction(float(c32[k])) + Fraction(float(c32[k + 1]))) / 2
            m32 = np.float32(float(mid))
            for v in (m32, np.nextafter(m32, np.float32(2)), np.nextafter(m32, np.float32(-2))):
                xs += [float(v), -float(v)]
    xs += list(synth.rng(91).uniform(-1, 1, 4000).astype(np.float32).astype(float))
    for x in xs:
        assert oracle.fp4_nearest_code(x) == _fp4_brute(x), x
    # the one exactly representable midpoint (half of the fp32 level 1/12) ties to zero, keeping the sign
    half = float(np.float32(c32[1]) / np.float32(2))
    assert oracle.fp4_nearest_code(half) == 0 and oracle.fp4_nearest_code(-half) == 8


def test_fp4_quantize_block_rules_and_round_trip():
    w = synth.normal_weights((64 * 40 + 17,), 92)
    w[64:128] = 0.0                # all-zero block -> +0 codes, absmax 0
    w[128:192] = -0.0
    w[200] = -0.0                  # a signed zero inside a normal block keeps its sign
    p, a = oracle.fp4_quantize(w, 64)
    codes = np.stack([p >> 4, p & 15], axis=1).reshape(-1)[:w.size]
    assert np.all(codes[64:192] == 0) and a[1] == 0 and a[2] == 0
    assert codes[200] == 8
    blocks = [(b * 64, min(b * 64 + 64, w.size)) for b in range(len(a))]
    for b, (lo, hi) in enumerate(blocks):  # the block's largest magnitude maps to +-1 (pattern 7 or 15)
        if a[b] > 0:
            j = lo + int(np.argmax(np.abs(w[lo:hi])))
            assert codes[j] == (15 if w[j] < 0 else 7)
    assert (p[-1] & 15) == 0  # odd tail: the partner is +0
    for i in range(0, w.size, 37):  # brute force on the same inputs
        if a[i // 64] > 0:
            assert codes[i] == _fp4_brute(float(np.float32(w[i]) / np.float32(a[i // 64])))
    # dequantize(quantize) is a fixed point: quantizing the dequantized tensor gives the same codes and scales
    d = oracle.fp4_dequantize(p, a, w.size, 64, "f32")
    p2, a2 = oracle.fp4_quantize(d, 64)
    assert np.array_equal(p2, p) and np.array_equal(a2, a)
    _, c32 = oracle.fp4_codebook()
    assert np.array_equal(d, (c32[codes] * np.repeat(a, 64)[:w.size]).astype(np.float32))


def test_fp4_bf16_input_and_output():
    bits = synth.normal_weights((64 * 8,), 93, dtype="bf16")
    p, a = oracle.fp4_quantize(bits, 64)
    pf, af = oracle.fp4_quantize(synth.bf16_bits_to_f32(bits), 64)
    assert np.array_equal(p, pf) and np.array_equal(a, af)  # widening bf16 to fp32 is exact
    d16 = oracle.fp4_dequantize(p, a, bits.size, 64, "bf16")
    d32 = oracle.fp4_dequantize(p, a, bits.size, 64, "f32")
    assert np.array_equal(d16, synth.f32_to_bf16_bits(d32))


def test_fp4_matmul_one_hot_and_numpy():
    """one-hot activations read bf16_rn(fp4[code] * a) back exactly; random activations match a numpy product"""
    N, K = 32, 192
    w = synth.normal_weights((N, K), 94)
    p, a = oracle.fp4_quantize(w, 64)
    wc = synth.bf16_bits_to_f32(oracle.fp4_dequantize(p, a, N * K, 64, "bf16")).reshape(N, K)
    ks = [0, 63, 64, 191]
    eye = synth.f32_to_bf16_bits(np.eye(K, dtype=np.float32)[ks])
    assert np.array_equal(oracle.fp4_matmul(p, a, N, K, eye), wc[:, ks].T.astype(np.float64))
    x = synth.activations((3, K), 95)
    ref = synth.bf16_bits_to_f32(x).astype(np.float64) @ wc.astype(np.float64).T
    assert np.allclose(oracle.fp4_matmul(p, a, N, K, x), ref, rtol=1e-12, atol=1e-15)
    # the NF4 and FP4 products of the same weight differ (different levels), so the code book is really swapped
    pn, an = oracle.quantize(w, 64)
    assert not np.allclose(oracle.matmul(pn, an, N, K, x), ref)


# ---------------------------------------------------------------- block sizes other than 64

@pytest.mark.parametrize("bs", [32, 128, 256, 4096])
def test_other_blocksizes_quantize_dequantize_matmul(bs):
    """the blockwise rules at other block sizes (the pages give 64 only as an example size): absmax per block
    equals numpy's max |w| per block, the block's largest element maps to +-1, every code is the brute-force
    nearest level, and dequantize / matmul follow from them"""
    N, K = 16, 4096
    w = synth.normal_weights((N * K + 7,), 96 + bs)  # ragged last block
    p, a = oracle.quantize(w, bs)
    nb = (w.size + bs - 1) // bs
    pad = np.zeros(nb * bs, np.float32)
    pad[:w.size] = w
    assert np.array_equal(a, np.abs(pad.reshape(nb, bs)).max(axis=1))
    codes = np.stack([p >> 4, p & 15], axis=1).reshape(-1)[:w.size]
    _, c32 = oracle.codebook()
    for b in range(0, nb, max(1, nb // 40)):
        lo, hi = b * bs, min(b * bs + bs, w.size)
        j = lo + int(np.argmax(np.abs(w[lo:hi])))
        assert codes[j] == (0 if w[j] < 0 else 15)
    for i in range(0, w.size, 997):
        x = np.float32(w[i]) / np.float32(a[i // bs])
        d = [abs(Fraction(float(x)) - Fraction(float(c))) for c in c32]
        assert codes[i] == min(range(16), key=lambda k: (d[k], k))
    d32 = oracle.dequantize(p, a, w.size, bs, "f32")
    assert np.array_equal(d32, (c32[codes] * np.repeat(a, bs)[:w.size]).astype(np.float32))
    pm, am = oracle.quantize(w[:N * K], bs)
    x = synth.activations((2, K), 97)
    wc = synth.bf16_bits_to_f32(oracle.dequantize(pm, am, N * K, bs, "bf16")).reshape(N, K)
    ref = synth.bf16_bits_to_f32(x).astype(np.float64) @ wc.astype(np.float64).T
    assert np.allclose(oracle.matmul(pm, am, N, K, x, bs), ref, rtol=1e-12, atol=1e-15)
