"""ctypes view of libnf4.so (the C ABI declared in include/nf4.h).

No fallback exists: if the shared library cannot be loaded, importing this
module raises, and every call that needs a GPU fails with the library's status.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnf4.so")

NF4_OK = 0
STATUS_NAMES = {0: "NF4_OK", 1: "NF4_ERR_INVALID_ARG", 2: "NF4_ERR_MISALIGNED", 3: "NF4_ERR_UNSUPPORTED",
                4: "NF4_ERR_ARCH", 5: "NF4_ERR_CUDA", 6: "NF4_ERR_TIMEOUT"}
NF4_F32, NF4_BF16 = 0, 1
NF4_DQ_E4M3, NF4_DQ_INT8 = 0, 1
NF4_QUANT_NF4, NF4_QUANT_FP4 = 0, 1

# every symbol include/nf4.h declares: name -> (restype, argtypes)
P = ctypes.c_void_p
I32 = ctypes.c_int32
I64 = ctypes.c_int64
SZ = ctypes.c_size_t


class NF4Weight(ctypes.Structure):
    """Mirror of the C struct nf4_weight."""
    _fields_ = [("packed", P), ("absmax", P), ("absmax_q", P), ("absmax_scale", P), ("absmax_mean", P),
                ("rows", I64), ("cols", I64), ("blocksize", I32), ("dq_blocksize", I32), ("dq_code", I32),
                ("quant_type", I32)]


class NF4Lora(ctypes.Structure):
    """Mirror of the C struct nf4_lora."""
    _fields_ = [("down", P), ("up", P), ("r", I32), ("scale", ctypes.c_float)]


SIGNATURES = {
    "nf4_quantize": (ctypes.c_int, [P, I32, I64, I32, P, P, P]),
    "nf4_quantize_typed": (ctypes.c_int, [P, I32, I64, I32, I32, P, P, P]),
    "nf4_double_quant": (ctypes.c_int, [P, I64, I32, I32, P, P, P, P, SZ, P]),
    "nf4_double_quant_workspace_bytes": (SZ, [I64]),
    "nf4_double_quant_noalloc": (ctypes.c_int, [P, I64, I32, I32, P, P, P, P]),
    "nf4_quantize_many": (ctypes.c_int, [ctypes.POINTER(P), ctypes.POINTER(I64), I32, I32, I32, I32, ctypes.POINTER(P),
                                         ctypes.POINTER(P), P]),
    "nf4_double_quant_many": (ctypes.c_int, [ctypes.POINTER(P), ctypes.POINTER(I64), I32, I32, I32, ctypes.POINTER(P),
                                             ctypes.POINTER(P), ctypes.POINTER(P), P, SZ, P]),
    "nf4_double_quant_many_workspace_bytes": (SZ, [I32]),
    "nf4_dequantize": (ctypes.c_int, [ctypes.POINTER(NF4Weight), P, I32, P]),
    "nf4_gemv": (ctypes.c_int, [ctypes.POINTER(NF4Weight), P, I32, P, P]),
    "nf4_gemv_grouped": (ctypes.c_int, [ctypes.POINTER(ctypes.POINTER(NF4Weight)), I32, P, I32, ctypes.POINTER(P), P]),
    "nf4_gemv_stream": (ctypes.c_int, [ctypes.POINTER(NF4Weight), ctypes.POINTER(P), ctypes.POINTER(P), I32, I32, P]),
    "nf4_gemm": (ctypes.c_int, [ctypes.POINTER(NF4Weight), P, I64, P, P, SZ, P]),
    "nf4_gemm_workspace_bytes": (SZ, [ctypes.POINTER(NF4Weight), I64]),
    "nf4_gemm_lora": (ctypes.c_int, [ctypes.POINTER(NF4Weight), ctypes.POINTER(NF4Lora), P, I64, P, P, SZ, P]),
    "nf4_gemm_lora_workspace_bytes": (SZ, [ctypes.POINTER(NF4Weight), I64]),
    "nf4_gemm_dx": (ctypes.c_int, [ctypes.POINTER(NF4Weight), P, I64, P, P, SZ, P]),
    "nf4_gemm_dx_workspace_bytes": (SZ, [ctypes.POINTER(NF4Weight), I64]),
    "nf4_storage_bytes": (SZ, [I64, I32, I32, I32]),
    "nf4_check_device_error": (ctypes.c_int, [P]),
    "nf4_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "nf4_code_table": (None, [ctypes.POINTER(ctypes.c_float)]),
    "nf4_device_supported": (I32, []),
    "nf4_kernel_launches": (ctypes.c_uint64, []),
    "nf4_selftest_wait_timeout": (ctypes.c_int, [P]),
}

_lib = None


def load():
    """Load libnf4.so (building it first if the sources are newer)."""
    global _lib
    if _lib is not None:
        return _lib
    from . import build
    if build.stale():
        build.build()
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libnf4.so not found at {LIB_PATH}; build it with python -m qlora_block_absmax_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


class NF4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


def check(status: int, what: str) -> None:
    if status != NF4_OK:
        raise NF4Error(status, what)
