"""The C-ABI library loads on a machine without a GPU, exports every function
include/nf4.h declares, and rejects bad arguments on the host before touching
CUDA.  No compute calls here."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from qlora_block_absmax_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "nf4.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nf4_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return _lib.load()


def test_every_declared_symbol_is_exported_and_bound(lib):
    names = declared_functions()
    assert len(names) >= 12
    for name in names:
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_status_strings(lib):
    for code, name in _lib.STATUS_NAMES.items():
        assert lib.nf4_status_string(code).decode() == name


def test_code_table_matches_oracle_bitwise(lib):
    buf = (ctypes.c_float * 16)()
    lib.nf4_code_table(buf)
    _, c32 = oracle.codebook()
    assert np.array_equal(np.array(buf[:], np.float32).view(np.uint32), c32.view(np.uint32))


def test_storage_bytes(lib):
    n = 4096 * 4096
    nb = n // 64
    assert lib.nf4_storage_bytes(n, 64, 0, 256) == n // 2 + 4 * nb
    assert lib.nf4_storage_bytes(n, 64, 1, 256) == n // 2 + nb + 4 * (nb // 256) + 4
    assert lib.nf4_storage_bytes(65, 64, 1, 256) == 33 + 2 + 4 + 4
    assert lib.nf4_storage_bytes(0, 64, 1, 256) == 0


def weight(rows=128, cols=128, packed=0x1000, absmax=0x2000, q=0, scale=0, mean=0, bs=64, dqbs=256, code=0):
    return _lib.NF4Weight(packed, absmax, q, scale, mean, rows, cols, bs, dqbs, code)


def test_host_validation_before_cuda(lib):
    E = {v: k for k, v in _lib.STATUS_NAMES.items()}
    s = None
    # quantize
    assert lib.nf4_quantize(0x1000, 0, -1, 64, 0x2000, 0x3000, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_quantize(0x1000, 7, 10, 64, 0x2000, 0x3000, s) == E["NF4_ERR_INVALID_ARG"]
    for bs in (16, 48, 512):  # level-1 sizes are 32, 64, 128 and 256
        assert lib.nf4_quantize(0x1000, 0, 10, bs, 0x2000, 0x3000, s) == E["NF4_ERR_UNSUPPORTED"]
    assert lib.nf4_quantize(0x1000, 0, 0, 64, 0x2000, 0x3000, s) == E["NF4_OK"]  # empty: nothing launched
    assert lib.nf4_quantize(None, 0, 10, 64, 0x2000, 0x3000, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_quantize(0x1008, 0, 10, 64, 0x2000, 0x3000, s) == E["NF4_ERR_MISALIGNED"]
    # double quant
    assert lib.nf4_double_quant(0x1000, 10, 128, 0, 0x2000, 0x3000, 0x4000, 0x5000, 256, s) == E["NF4_ERR_UNSUPPORTED"]
    assert lib.nf4_double_quant(0x1000, 10, 256, 5, 0x2000, 0x3000, 0x4000, 0x5000, 256, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_double_quant(0x1000, 10, 256, 0, 0x2000, 0x3000, 0x4000, 0x5000, 8, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_double_quant(0x1000, 0, 256, 0, 0x2000, 0x3000, 0x4000, 0x5000, 256, s) == E["NF4_OK"]
    too_many = 2 ** 31  # one past NF4_DQ_MAX_NB: the exact-sum limbs would no longer be exact
    assert lib.nf4_double_quant(0x1000, too_many, 256, 0, 0x2000, 0x3000, 0x4000, 0x5000, 256, s) == \
        E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_double_quant_noalloc(0x1000, too_many, 256, 0, 0x2000, 0x3000, 0x4000, s) == \
        E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_double_quant_workspace_bytes(1 << 20) >= 128
    # the many-array call checks every array before it touches the device
    P = ctypes.c_void_p
    one = lambda *v: (P * len(v))(*v)  # noqa: E731
    nb = lambda *v: (ctypes.c_int64 * len(v))(*v)  # noqa: E731
    dqm = lib.nf4_double_quant_many
    assert dqm(one(0x1000), nb(10), 0, 256, 0, one(0x2000), one(0x3000), one(0x4000), 0x5000, 4096, s) == \
        E["NF4_ERR_INVALID_ARG"]
    assert dqm(one(0x1000), nb(10), 257, 256, 0, one(0x2000), one(0x3000), one(0x4000), 0x5000, 1 << 20, s) == \
        E["NF4_ERR_INVALID_ARG"]
    assert dqm(one(0x1000), nb(10), 1, 128, 0, one(0x2000), one(0x3000), one(0x4000), 0x5000, 4096, s) == \
        E["NF4_ERR_UNSUPPORTED"]
    assert dqm(one(0x1000), nb(10), 1, 256, 7, one(0x2000), one(0x3000), one(0x4000), 0x5000, 4096, s) == \
        E["NF4_ERR_INVALID_ARG"]
    assert dqm(one(0x1000), nb(10), 1, 256, 0, one(0x2000), one(0x3000), one(0x4000), 0x5000, 16, s) == \
        E["NF4_ERR_INVALID_ARG"]  # workspace smaller than one record
    assert dqm(one(0x1000, 0x1004), nb(10, 10), 2, 256, 0, one(0x2000, 0x2100), one(0x3000, 0x3100),
               one(0x4000, 0x4100), 0x5000, 4096, s) == E["NF4_ERR_MISALIGNED"]  # second array misaligned
    assert dqm(one(0x1000), nb(-1), 1, 256, 0, one(0x2000), one(0x3000), one(0x4000), 0x5000, 4096, s) == \
        E["NF4_ERR_INVALID_ARG"]
    assert dqm(one(0x1000), nb(0), 1, 256, 0, one(0x2000), one(0x3000), one(0x4000), 0x5000, 4096, s) == E["NF4_OK"]
    assert lib.nf4_double_quant_many_workspace_bytes(3) == 3 * 128
    qm = lib.nf4_quantize_many
    assert qm(one(0x1000), nb(10), 0, 0, 64, 0, one(0x2000), one(0x3000), s) == E["NF4_ERR_INVALID_ARG"]
    assert qm(one(0x1000), nb(10), 257, 0, 64, 0, one(0x2000), one(0x3000), s) == E["NF4_ERR_INVALID_ARG"]
    assert qm(one(0x1000), nb(10), 1, 7, 64, 0, one(0x2000), one(0x3000), s) == E["NF4_ERR_INVALID_ARG"]
    assert qm(one(0x1000), nb(10), 1, 0, 48, 0, one(0x2000), one(0x3000), s) == E["NF4_ERR_UNSUPPORTED"]
    assert qm(one(0x1000), nb(10), 1, 0, 64, 9, one(0x2000), one(0x3000), s) == E["NF4_ERR_INVALID_ARG"]
    assert qm(one(0x1000, 0x1008), nb(10, 10), 2, 0, 64, 0, one(0x2000, 0x2100), one(0x3000, 0x3100), s) == \
        E["NF4_ERR_MISALIGNED"]  # second source misaligned
    assert qm(one(0x1000), nb(-1), 1, 0, 64, 0, one(0x2000), one(0x3000), s) == E["NF4_ERR_INVALID_ARG"]
    assert qm(one(0x1000), nb(0), 1, 0, 64, 0, one(0x2000), one(0x3000), s) == E["NF4_OK"]
    assert lib.nf4_double_quant_many_workspace_bytes(0) == 0 and lib.nf4_double_quant_many_workspace_bytes(257) == 0
    # weight descriptor checks
    w = weight(bs=48)
    assert lib.nf4_dequantize(ctypes.byref(w), 0x9000, 0, s) == E["NF4_ERR_UNSUPPORTED"]
    w = weight(packed=0x1001)
    assert lib.nf4_dequantize(ctypes.byref(w), 0x9000, 0, s) == E["NF4_ERR_MISALIGNED"]
    w = weight(absmax=0)  # neither plain scales nor a double-quant record
    assert lib.nf4_dequantize(ctypes.byref(w), 0x9000, 0, s) == E["NF4_ERR_INVALID_ARG"]
    w = weight(absmax=0, q=0x3000, scale=0x4000, mean=0x5000, code=9)
    assert lib.nf4_dequantize(ctypes.byref(w), 0x9000, 0, s) == E["NF4_ERR_INVALID_ARG"]
    w = weight()
    assert lib.nf4_dequantize(ctypes.byref(w), 0x9000, 4, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_dequantize(None, 0x9000, 0, s) == E["NF4_ERR_INVALID_ARG"]
    # gemv / gemm shape rules
    assert lib.nf4_gemv(ctypes.byref(w), 0x9000, 9, 0xa000, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_gemv(ctypes.byref(w), 0x9000, 0, 0xa000, s) == E["NF4_ERR_INVALID_ARG"]
    w = weight(cols=96)
    assert lib.nf4_gemv(ctypes.byref(w), 0x9000, 1, 0xa000, s) == E["NF4_ERR_UNSUPPORTED"]
    w = weight(rows=120)
    assert lib.nf4_gemv(ctypes.byref(w), 0x9000, 1, 0xa000, s) == E["NF4_ERR_UNSUPPORTED"]
    w = weight(rows=112)
    assert lib.nf4_gemm(ctypes.byref(w), 0x9000, 4, 0xa000, None, 0, s) == E["NF4_ERR_UNSUPPORTED"]
    w = weight()
    assert lib.nf4_gemm(ctypes.byref(w), 0x9000, -1, 0xa000, None, 0, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_gemm(ctypes.byref(w), 0x9000, 0, 0xa000, None, 0, s) == E["NF4_OK"]
    assert lib.nf4_gemm(ctypes.byref(w), 0x9008, 4, 0xa000, None, 0, s) == E["NF4_ERR_MISALIGNED"]


def test_device_query_without_gpu_is_safe(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    assert lib.nf4_device_supported() == 0


def test_host_validation_new_entry_points(lib):
    """nf4_gemm_dx, nf4_gemm_lora and nf4_gemv_grouped reject bad arguments on the host, before any CUDA call"""
    E = {v: k for k, v in _lib.STATUS_NAMES.items()}
    s = None
    w = weight(rows=128, cols=256)
    # input gradient: rows % 64, cols % 128, m >= 0, alignment, workspace
    assert lib.nf4_gemm_dx(ctypes.byref(weight(rows=96, cols=256)), 0x9000, 4, 0xa000, None, 0, s) == \
        E["NF4_ERR_UNSUPPORTED"]
    assert lib.nf4_gemm_dx(ctypes.byref(weight(rows=128, cols=192)), 0x9000, 4, 0xa000, None, 0, s) == \
        E["NF4_ERR_UNSUPPORTED"]
    assert lib.nf4_gemm_dx(ctypes.byref(w), 0x9000, -1, 0xa000, None, 0, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_gemm_dx(ctypes.byref(w), 0x9000, 0, 0xa000, None, 0, s) == E["NF4_OK"]
    assert lib.nf4_gemm_dx(ctypes.byref(w), 0x9004, 4, 0xa000, None, 0, s) == E["NF4_ERR_MISALIGNED"]
    assert lib.nf4_gemm_dx(ctypes.byref(w), None, 4, 0xa000, None, 0, s) == E["NF4_ERR_INVALID_ARG"]
    # adapter: r in {16, 32}, finite scale, workspace present and large enough
    lo = _lib.NF4Lora(0xb000, 0xc000, 16, 2.0)
    assert lib.nf4_gemm_lora(ctypes.byref(w), None, 0x9000, 4, 0xa000, 0xd000, 1 << 20, s) == E["NF4_ERR_INVALID_ARG"]
    bad_r = _lib.NF4Lora(0xb000, 0xc000, 8, 2.0)
    assert lib.nf4_gemm_lora(ctypes.byref(w), ctypes.byref(bad_r), 0x9000, 4, 0xa000, 0xd000, 1 << 20, s) == \
        E["NF4_ERR_UNSUPPORTED"]
    nan_s = _lib.NF4Lora(0xb000, 0xc000, 16, float("nan"))
    assert lib.nf4_gemm_lora(ctypes.byref(w), ctypes.byref(nan_s), 0x9000, 4, 0xa000, 0xd000, 1 << 20, s) == \
        E["NF4_ERR_INVALID_ARG"]
    inf_s = _lib.NF4Lora(0xb000, 0xc000, 16, float("inf"))
    assert lib.nf4_gemm_lora(ctypes.byref(w), ctypes.byref(inf_s), 0x9000, 4, 0xa000, 0xd000, 1 << 20, s) == \
        E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_gemm_lora(ctypes.byref(w), ctypes.byref(lo), 0x9000, 4, 0xa000, None, 0, s) == \
        E["NF4_ERR_INVALID_ARG"]
    unaligned = _lib.NF4Lora(0xb008, 0xc000, 16, 2.0)
    assert lib.nf4_gemm_lora(ctypes.byref(w), ctypes.byref(unaligned), 0x9000, 4, 0xa000, 0xd000, 1 << 20, s) == \
        E["NF4_ERR_MISALIGNED"]
    assert lib.nf4_gemm_lora(ctypes.byref(w), ctypes.byref(lo), 0x9000, 0, 0xa000, None, 0, s) == E["NF4_OK"]
    # grouped GEMV: 1..4 weights, equal cols and scale kind, batch 1..8
    ws = (ctypes.POINTER(_lib.NF4Weight) * 5)(*[ctypes.pointer(weight()) for _ in range(5)])
    ys = (ctypes.c_void_p * 5)(*[0xa000] * 5)
    assert lib.nf4_gemv_grouped(ws, 0, 0x9000, 1, ys, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_gemv_grouped(ws, 5, 0x9000, 1, ys, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_gemv_grouped(ws, 2, 0x9000, 9, ys, s) == E["NF4_ERR_INVALID_ARG"]
    mixed = (ctypes.POINTER(_lib.NF4Weight) * 2)(ctypes.pointer(weight(cols=128)), ctypes.pointer(weight(cols=256)))
    assert lib.nf4_gemv_grouped(mixed, 2, 0x9000, 1, ys, s) == E["NF4_ERR_INVALID_ARG"]
    kinds = (ctypes.POINTER(_lib.NF4Weight) * 2)(
        ctypes.pointer(weight()), ctypes.pointer(weight(absmax=0, q=0x3000, scale=0x4000, mean=0x5000)))
    assert lib.nf4_gemv_grouped(kinds, 2, 0x9000, 1, ys, s) == E["NF4_ERR_INVALID_ARG"]
    odd = (ctypes.POINTER(_lib.NF4Weight) * 2)(ctypes.pointer(weight()), ctypes.pointer(weight(rows=40)))
    assert lib.nf4_gemv_grouped(odd, 2, 0x9000, 1, ys, s) == E["NF4_ERR_UNSUPPORTED"]
    assert lib.nf4_gemv_grouped(ws, 2, 0x9008, 1, ys, s) == E["NF4_ERR_MISALIGNED"]


def test_plain_c_client(tmp_path):
    """the header compiles as C and a C program linked against libnf4.so gets the documented host-side results"""
    import os
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(_lib.load()._name)
    exe = str(tmp_path / "abi_check")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(root, "include"),
                    os.path.join(root, "tests", "c_abi", "abi_check.c"), "-L", libdir, "-lnf4",
                    "-Wl,-rpath," + libdir, "-lm", "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr


def test_host_validation_gemv_stream(lib):
    """nf4_gemv_stream rejects bad arguments on the host, before any CUDA call: count 1..256, batch 1..8,
    per-weight shape rules, null and misaligned pointers; a list of empty weights launches nothing"""
    E = {v: k for k, v in _lib.STATUS_NAMES.items()}
    s = None
    n = 257
    ws = (_lib.NF4Weight * n)(*[weight() for _ in range(n)])
    xs = (ctypes.c_void_p * n)(*[0x9000] * n)
    ys = (ctypes.c_void_p * n)(*[0xa000] * n)
    assert lib.nf4_gemv_stream(ws, xs, ys, 0, 1, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_gemv_stream(ws, xs, ys, 257, 1, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_gemv_stream(ws, xs, ys, 2, 0, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_gemv_stream(ws, xs, ys, 2, 9, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_gemv_stream(None, xs, ys, 2, 1, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_gemv_stream(ws, None, ys, 2, 1, s) == E["NF4_ERR_INVALID_ARG"]
    assert lib.nf4_gemv_stream(ws, xs, None, 2, 1, s) == E["NF4_ERR_INVALID_ARG"]
    mixed = (_lib.NF4Weight * 3)(weight(), weight(cols=96), weight())
    assert lib.nf4_gemv_stream(mixed, xs, ys, 3, 1, s) == E["NF4_ERR_UNSUPPORTED"]
    mixed = (_lib.NF4Weight * 2)(weight(), weight(rows=40))
    assert lib.nf4_gemv_stream(mixed, xs, ys, 2, 1, s) == E["NF4_ERR_UNSUPPORTED"]
    mixed = (_lib.NF4Weight * 2)(weight(), weight(bs=128))
    assert lib.nf4_gemv_stream(mixed, xs, ys, 2, 1, s) == E["NF4_ERR_UNSUPPORTED"]
    mixed = (_lib.NF4Weight * 2)(weight(), weight(absmax=0))
    assert lib.nf4_gemv_stream(mixed, xs, ys, 2, 1, s) == E["NF4_ERR_INVALID_ARG"]
    xs_bad = (ctypes.c_void_p * 2)(0x9000, 0x9008)
    assert lib.nf4_gemv_stream(ws, xs_bad, ys, 2, 1, s) == E["NF4_ERR_MISALIGNED"]
    ys_bad = (ctypes.c_void_p * 2)(0xa000, 0xa002)
    assert lib.nf4_gemv_stream(ws, xs, ys_bad, 2, 1, s) == E["NF4_ERR_MISALIGNED"]
    xs_null = (ctypes.c_void_p * 2)(0x9000, None)
    assert lib.nf4_gemv_stream(ws, xs_null, ys, 2, 1, s) == E["NF4_ERR_INVALID_ARG"]
    empty = (_lib.NF4Weight * 2)(weight(rows=0), weight(cols=0))
    assert lib.nf4_gemv_stream(empty, xs_null, ys, 2, 1, s) == E["NF4_OK"]  # nothing to compute, nothing launched
