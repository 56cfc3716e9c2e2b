"""Plain CPU oracle for NF4 quantization, double quantization, dequantization
and the 4-bit x bf16 matmul -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package.  The product library (``qlora_block_absmax_b200``)
never imports it and shares no code with it.

The arithmetic lives in ``nf4_oracle.c`` (plain C, -ffp-contract=off); this
module compiles it with gcc on first use and wraps it for numpy arrays.  Arrays
of bf16 values are passed as ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nf4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

DQ_E4M3 = 0
DQ_INT8 = 1


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (gcc, OpenMP, no FMA contraction)."""
    with _lock:
        stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < max(
            os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "nf4_oracle.h")))
        if force or stale:
            tmp = _LIB + f".tmp{os.getpid()}"
            cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                   "-fexcess-precision=standard", "-fopenmp", "-fPIC", "-shared",
                   "-o", tmp, _SRC, "-lm"]
            subprocess.run(cmd, check=True)
            os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    I32 = ctypes.c_int32
    sig = {
        "oracle_nf4_codebook": (None, [P, P]),
        "oracle_bf16_rn": (ctypes.c_uint16, [ctypes.c_float]),
        "oracle_nf4_quantize_f32": (None, [P, I64, I32, P, P]),
        "oracle_nf4_quantize_bf16": (None, [P, I64, I32, P, P]),
        "oracle_nf4_nearest_code": (ctypes.c_int, [ctypes.c_float]),
        "oracle_exact_sum_f32": (ctypes.c_double, [P, I64]),
        "oracle_e4m3_decode": (ctypes.c_float, [ctypes.c_uint8]),
        "oracle_e4m3_encode_satfinite": (ctypes.c_uint8, [ctypes.c_float]),
        "oracle_blockwise_8bit": (None, [P, I64, I32, ctypes.c_int, P, P]),
        "oracle_blockwise_8bit_value": (ctypes.c_float, [ctypes.c_uint8, ctypes.c_float, ctypes.c_int]),
        "oracle_nf4_double_quant": (None, [P, I64, I32, ctypes.c_int, P, P, P]),
        "oracle_absmax_reconstruct": (None, [P, P, ctypes.c_float, I64, I32, ctypes.c_int, P]),
        "oracle_nf4_dequantize_f32": (None, [P, P, I64, I32, P]),
        "oracle_nf4_dequantize_bf16": (None, [P, P, I64, I32, P]),
        "oracle_nf4_matmul": (None, [P, P, I64, I64, I32, P, I64, P]),
        "oracle_nf4_matmul_sampled": (None, [P, P, I64, I64, I32, P, I64, P, P, I64, P]),
        "oracle_nf4_matmul_dx": (None, [P, P, I64, I64, I32, P, I64, P]),
        "oracle_nf4_matmul_dx_sampled": (None, [P, P, I64, I64, I32, P, I64, P, P, I64, P]),
        "oracle_lora_down": (None, [P, I64, I64, P, I32, ctypes.c_float, P]),
        "oracle_nf4_matmul_lora": (None, [P, P, I64, I64, I32, P, I64, P, P, I32, ctypes.c_float, P]),
        "oracle_nf4_matmul_lora_sampled": (None, [P, P, I64, I64, I32, P, P, P, I32, P, P, I64, P]),
        "oracle_fp4_codebook": (None, [P, P]),
        "oracle_fp4_nearest_code": (ctypes.c_int, [ctypes.c_float]),
        "oracle_fp4_quantize_f32": (None, [P, I64, I32, P, P]),
        "oracle_fp4_quantize_bf16": (None, [P, I64, I32, P, P]),
        "oracle_fp4_dequantize_f32": (None, [P, P, I64, I32, P]),
        "oracle_fp4_dequantize_bf16": (None, [P, P, I64, I32, P]),
        "oracle_fp4_matmul": (None, [P, P, I64, I64, I32, P, I64, P]),
        "oracle_set_threads": (None, [ctypes.c_int]),
        "oracle_get_threads": (ctypes.c_int, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_load().oracle_get_threads())


def codebook():
    """(fp64 levels, fp32 levels), ascending, 16 each."""
    c64 = np.zeros(16, np.float64)
    c32 = np.zeros(16, np.float32)
    _load().oracle_nf4_codebook(_p(c64), _p(c32))
    return c64, c32


def bf16_rn(v: float) -> int:
    return int(_load().oracle_bf16_rn(float(v)))


def nearest_code(x: float) -> int:
    return int(_load().oracle_nf4_nearest_code(float(x)))


def quantize(w: np.ndarray, blocksize: int = 64):
    """w: float32 array, or uint16 array of bf16 bit patterns -> (packed u8, absmax f32)."""
    w = np.ascontiguousarray(w).reshape(-1)
    n = w.size
    packed = np.zeros((n + 1) // 2, np.uint8)
    absmax = np.zeros((n + blocksize - 1) // blocksize, np.float32)
    if w.dtype == np.float32:
        _load().oracle_nf4_quantize_f32(_p(w), n, blocksize, _p(packed), _p(absmax))
    elif w.dtype == np.uint16:
        _load().oracle_nf4_quantize_bf16(_p(w), n, blocksize, _p(packed), _p(absmax))
    else:
        raise TypeError("quantize takes float32 or bf16 bit patterns (uint16)")
    return packed, absmax


def exact_sum(a: np.ndarray) -> float:
    a = np.ascontiguousarray(a, dtype=np.float32).reshape(-1)
    return float(_load().oracle_exact_sum_f32(_p(a), a.size))


def e4m3_decode(code: int) -> float:
    return float(_load().oracle_e4m3_decode(int(code)))


def e4m3_encode(y: float) -> int:
    return int(_load().oracle_e4m3_encode_satfinite(float(y)))


def blockwise_8bit(v: np.ndarray, blocksize: int, code: int):
    v = np.ascontiguousarray(v, dtype=np.float32).reshape(-1)
    q = np.zeros(v.size, np.uint8)
    scale = np.zeros((v.size + blocksize - 1) // blocksize, np.float32)
    _load().oracle_blockwise_8bit(_p(v), v.size, blocksize, code, _p(q), _p(scale))
    return q, scale


def blockwise_8bit_value(q: int, scale: float, code: int) -> float:
    return float(_load().oracle_blockwise_8bit_value(int(q), float(scale), int(code)))


def double_quant(absmax: np.ndarray, dq_blocksize: int = 256, code: int = DQ_E4M3):
    """-> (q u8 [nb], scale f32 [ceil(nb/dq)], mean float)"""
    a = np.ascontiguousarray(absmax, dtype=np.float32).reshape(-1)
    nb = a.size
    q = np.zeros(nb, np.uint8)
    scale = np.zeros((nb + dq_blocksize - 1) // dq_blocksize, np.float32)
    mean = np.zeros(1, np.float32)
    _load().oracle_nf4_double_quant(_p(a), nb, dq_blocksize, code, _p(q), _p(scale), _p(mean))
    return q, scale, float(mean[0])


def absmax_reconstruct(q: np.ndarray, scale: np.ndarray, mean: float, dq_blocksize: int = 256,
                       code: int = DQ_E4M3) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8).reshape(-1)
    scale = np.ascontiguousarray(scale, dtype=np.float32).reshape(-1)
    out = np.zeros(q.size, np.float32)
    _load().oracle_absmax_reconstruct(_p(q), _p(scale), float(mean), q.size, dq_blocksize, code, _p(out))
    return out


def dequantize(packed: np.ndarray, absmax: np.ndarray, n: int, blocksize: int = 64,
               out_dtype: str = "f32") -> np.ndarray:
    """absmax: one fp32 scale per block (reconstructed when double-quantized).
    out_dtype 'f32' -> float32 array; 'bf16' -> uint16 bit patterns."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    absmax = np.ascontiguousarray(absmax, dtype=np.float32)
    if out_dtype == "f32":
        out = np.zeros(n, np.float32)
        _load().oracle_nf4_dequantize_f32(_p(packed), _p(absmax), n, blocksize, _p(out))
    elif out_dtype == "bf16":
        out = np.zeros(n, np.uint16)
        _load().oracle_nf4_dequantize_bf16(_p(packed), _p(absmax), n, blocksize, _p(out))
    else:
        raise ValueError(out_dtype)
    return out


def matmul(packed: np.ndarray, absmax: np.ndarray, N: int, K: int, x_bf16: np.ndarray,
           blocksize: int = 64) -> np.ndarray:
    """x_bf16: uint16 [B, K] -> fp64 y [B, N] = x . Wc^T, fp64 accumulation."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16).reshape(-1, K)
    B = x.shape[0]
    y = np.zeros((B, N), np.float64)
    _load().oracle_nf4_matmul(_p(np.ascontiguousarray(packed, dtype=np.uint8)),
                              _p(np.ascontiguousarray(absmax, dtype=np.float32)),
                              N, K, blocksize, _p(x), B, _p(y))
    return y


def matmul_sampled(packed: np.ndarray, absmax: np.ndarray, N: int, K: int, x_bf16: np.ndarray,
                   bs: np.ndarray, ns: np.ndarray, blocksize: int = 64) -> np.ndarray:
    """fp64 y at the given (b, n) coordinates only."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16).reshape(-1, K)
    bs = np.ascontiguousarray(bs, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    y = np.zeros(bs.size, np.float64)
    _load().oracle_nf4_matmul_sampled(_p(np.ascontiguousarray(packed, dtype=np.uint8)),
                                      _p(np.ascontiguousarray(absmax, dtype=np.float32)),
                                      N, K, blocksize, _p(x), x.shape[0], _p(bs), _p(ns), bs.size, _p(y))
    return y


def matmul_dx(packed: np.ndarray, absmax: np.ndarray, N: int, K: int, dy_bf16: np.ndarray,
              blocksize: int = 64) -> np.ndarray:
    """Input gradient of ``matmul``: dy_bf16 uint16 [B, N] -> fp64 dx [B, K] = dy . Wc,
    fp64 accumulation over n."""
    dy = np.ascontiguousarray(dy_bf16, dtype=np.uint16).reshape(-1, N)
    B = dy.shape[0]
    dx = np.zeros((B, K), np.float64)
    _load().oracle_nf4_matmul_dx(_p(np.ascontiguousarray(packed, dtype=np.uint8)),
                                 _p(np.ascontiguousarray(absmax, dtype=np.float32)),
                                 N, K, blocksize, _p(dy), B, _p(dx))
    return dx


def matmul_dx_sampled(packed: np.ndarray, absmax: np.ndarray, N: int, K: int, dy_bf16: np.ndarray,
                      bs: np.ndarray, ks: np.ndarray, blocksize: int = 64) -> np.ndarray:
    """fp64 dx at the given (b, k) coordinates only."""
    dy = np.ascontiguousarray(dy_bf16, dtype=np.uint16).reshape(-1, N)
    bs = np.ascontiguousarray(bs, dtype=np.int64)
    ks = np.ascontiguousarray(ks, dtype=np.int64)
    dx = np.zeros(bs.size, np.float64)
    _load().oracle_nf4_matmul_dx_sampled(_p(np.ascontiguousarray(packed, dtype=np.uint8)),
                                         _p(np.ascontiguousarray(absmax, dtype=np.float32)),
                                         N, K, blocksize, _p(dy), dy.shape[0], _p(bs), _p(ks), bs.size, _p(dx))
    return dx


def lora_down(x_bf16: np.ndarray, K: int, A_bf16: np.ndarray, r: int, scale: float) -> np.ndarray:
    """fp64 t [B, r] = scale * x . A^T (not rounded)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16).reshape(-1, K)
    A = np.ascontiguousarray(A_bf16, dtype=np.uint16).reshape(r, K)
    t = np.zeros((x.shape[0], r), np.float64)
    _load().oracle_lora_down(_p(x), x.shape[0], K, _p(A), r, float(scale), _p(t))
    return t


def matmul_lora(packed: np.ndarray, absmax: np.ndarray, N: int, K: int, x_bf16: np.ndarray, A_bf16: np.ndarray,
                B_bf16: np.ndarray, r: int, scale: float, blocksize: int = 64) -> np.ndarray:
    """fp64 y [B, N] = x . Wc^T + t . B^T with t = lora_down(x) (fp64, not rounded)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16).reshape(-1, K)
    A = np.ascontiguousarray(A_bf16, dtype=np.uint16).reshape(r, K)
    Bu = np.ascontiguousarray(B_bf16, dtype=np.uint16).reshape(N, r)
    y = np.zeros((x.shape[0], N), np.float64)
    _load().oracle_nf4_matmul_lora(_p(np.ascontiguousarray(packed, dtype=np.uint8)),
                                   _p(np.ascontiguousarray(absmax, dtype=np.float32)), N, K, blocksize, _p(x),
                                   x.shape[0], _p(A), _p(Bu), r, float(scale), _p(y))
    return y


def matmul_lora_sampled(packed: np.ndarray, absmax: np.ndarray, N: int, K: int, x_bf16: np.ndarray,
                        A_bf16: np.ndarray, B_bf16: np.ndarray, r: int, scale: float, bs: np.ndarray,
                        ns: np.ndarray, blocksize: int = 64) -> np.ndarray:
    """fp64 y of ``matmul_lora`` at the given (b, n) coordinates only."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16).reshape(-1, K)
    t = lora_down(x, K, A_bf16, r, scale)
    Bu = np.ascontiguousarray(B_bf16, dtype=np.uint16).reshape(N, r)
    bs = np.ascontiguousarray(bs, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    y = np.zeros(bs.size, np.float64)
    _load().oracle_nf4_matmul_lora_sampled(_p(np.ascontiguousarray(packed, dtype=np.uint8)),
                                           _p(np.ascontiguousarray(absmax, dtype=np.float32)), N, K, blocksize,
                                           _p(x), _p(t), _p(Bu), r, _p(bs), _p(ns), bs.size, _p(y))
    return y


# ---------------------------------------------------------------- FP4 (E2M1 / 6, stored as the bit pattern)

def fp4_codebook():
    """(fp64 levels, fp32 levels) indexed by the 4-bit pattern s e1 e0 m."""
    c64 = np.zeros(16, np.float64)
    c32 = np.zeros(16, np.float32)
    _load().oracle_fp4_codebook(_p(c64), _p(c32))
    return c64, c32


def fp4_nearest_code(x: float) -> int:
    return int(_load().oracle_fp4_nearest_code(float(x)))


def fp4_quantize(w: np.ndarray, blocksize: int = 64):
    """w: float32, or uint16 bf16 bit patterns -> (packed u8, absmax f32), FP4 codes."""
    w = np.ascontiguousarray(w).reshape(-1)
    n = w.size
    packed = np.zeros((n + 1) // 2, np.uint8)
    absmax = np.zeros((n + blocksize - 1) // blocksize, np.float32)
    if w.dtype == np.float32:
        _load().oracle_fp4_quantize_f32(_p(w), n, blocksize, _p(packed), _p(absmax))
    elif w.dtype == np.uint16:
        _load().oracle_fp4_quantize_bf16(_p(w), n, blocksize, _p(packed), _p(absmax))
    else:
        raise TypeError("fp4_quantize takes float32 or bf16 bit patterns (uint16)")
    return packed, absmax


def fp4_dequantize(packed: np.ndarray, absmax: np.ndarray, n: int, blocksize: int = 64,
                   out_dtype: str = "f32") -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    absmax = np.ascontiguousarray(absmax, dtype=np.float32)
    if out_dtype == "f32":
        out = np.zeros(n, np.float32)
        _load().oracle_fp4_dequantize_f32(_p(packed), _p(absmax), n, blocksize, _p(out))
    elif out_dtype == "bf16":
        out = np.zeros(n, np.uint16)
        _load().oracle_fp4_dequantize_bf16(_p(packed), _p(absmax), n, blocksize, _p(out))
    else:
        raise ValueError(out_dtype)
    return out


def fp4_matmul(packed: np.ndarray, absmax: np.ndarray, N: int, K: int, x_bf16: np.ndarray,
               blocksize: int = 64) -> np.ndarray:
    """x_bf16: uint16 [B, K] -> fp64 y [B, N] = x . Wc^T with FP4 levels."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16).reshape(-1, K)
    y = np.zeros((x.shape[0], N), np.float64)
    _load().oracle_fp4_matmul(_p(np.ascontiguousarray(packed, dtype=np.uint8)),
                              _p(np.ascontiguousarray(absmax, dtype=np.float32)), N, K, blocksize, _p(x),
                              x.shape[0], _p(y))
    return y
