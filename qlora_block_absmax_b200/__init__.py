"""qlora_block_absmax_b200 -- blockwise NF4 quantization with double
quantization, dequantization and the NF4-weight x bf16 matmul on B200.

This module only marshals torch tensors (device memory, the current stream)
into the C ABI of libnf4.so; every step of the computation runs in the
library's sm_100a kernels.  There is no CPU path.

Typical use:
    qw = quantize_weight(W)            # W: [N, K] bf16/fp32 CUDA tensor
    y = gemv(qw, x)                    # x: [B, K] bf16, B <= 8
    Y = gemm(qw, X)                    # X: [M, K] bf16
    W_hat = dequantize(qw, torch.bfloat16)
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib
from ._lib import NF4_BF16, NF4_DQ_E4M3, NF4_DQ_INT8, NF4_F32, NF4_QUANT_FP4, NF4_QUANT_NF4, NF4Error

__all__ = ["QuantizedWeight", "quantize", "double_quant", "quantize_weight", "dequantize", "gemv", "gemm",
           "storage_bytes", "gemm_workspace_bytes", "gemm_dx", "gemm_dx_workspace_bytes", "gemm_lora", "gemv_grouped", "gemv_stream",
           "double_quant_many", "quantize_many",
           "gemm_lora_workspace_bytes", "code_table", "check_device_error", "kernel_launches", "NF4Error", "library_path"]

BLOCKSIZE = 64
DQ_BLOCKSIZE = 256
_DQ_CODES = {"e4m3": NF4_DQ_E4M3, "int8": NF4_DQ_INT8}
_QUANT_TYPES = {"nf4": NF4_QUANT_NF4, "fp4": NF4_QUANT_FP4}


def library_path() -> str:
    _lib.load()
    return _lib.LIB_PATH


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream: Optional[torch.cuda.Stream] = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


@dataclass
class QuantizedWeight:
    """A weight [rows, cols] in NF4: packed codes plus either fp32 block
    scales (absmax) or the double-quantized record (absmax_q, absmax_scale,
    absmax_mean)."""
    packed: torch.Tensor
    rows: int
    cols: int
    absmax: Optional[torch.Tensor] = None
    absmax_q: Optional[torch.Tensor] = None
    absmax_scale: Optional[torch.Tensor] = None
    absmax_mean: Optional[torch.Tensor] = None
    dq_code: int = NF4_DQ_E4M3
    blocksize: int = BLOCKSIZE
    dq_blocksize: int = DQ_BLOCKSIZE
    quant_type: int = NF4_QUANT_NF4

    @property
    def double_quant(self) -> bool:
        return self.absmax is None

    def descriptor(self) -> _lib.NF4Weight:
        return _lib.NF4Weight(_ptr(self.packed), _ptr(self.absmax), _ptr(self.absmax_q), _ptr(self.absmax_scale),
                              _ptr(self.absmax_mean), self.rows, self.cols, self.blocksize, self.dq_blocksize,
                              self.dq_code, self.quant_type)

    def storage_bytes(self) -> int:
        return storage_bytes(self.rows * self.cols, self.double_quant)


def quantize(w: torch.Tensor, blocksize: int = BLOCKSIZE, out=None, stream=None, quant_type: str = "nf4"):
    """Level-1 4-bit quantization (NF4, or FP4 with quant_type="fp4") of a flattened fp32/bf16 tensor.
    Returns (packed uint8 [ceil(n/2)], absmax fp32 [ceil(n/blocksize)])."""
    _need_cuda(w, "w")
    if w.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("quantize takes float32 or bfloat16")
    n = w.numel()
    if out is None:
        packed = torch.empty((n + 1) // 2, dtype=torch.uint8, device=w.device)
        absmax = torch.empty((n + blocksize - 1) // blocksize, dtype=torch.float32, device=w.device)
    else:
        packed, absmax = out
    st = _lib.load().nf4_quantize_typed(_ptr(w), NF4_BF16 if w.dtype == torch.bfloat16 else NF4_F32, n, blocksize,
                                        _QUANT_TYPES[quant_type], _ptr(packed), _ptr(absmax), _stream(stream))
    _lib.check(st, "nf4_quantize_typed")
    return packed, absmax


def quantize_many(ws, blocksize: int = BLOCKSIZE, outs=None, stream=None, quant_type: str = "nf4") -> list:
    """quantize of up to 256 flattened tensors of one dtype (fp32 or bf16) in one launch.
    Returns [(packed, absmax)] per tensor, the same values quantize gives each one."""
    ws = list(ws)
    if not ws:
        raise ValueError("quantize_many takes at least one tensor")
    dt = ws[0].dtype
    for w in ws:
        _need_cuda(w, "w")
        if w.dtype != dt or dt not in (torch.float32, torch.bfloat16):
            raise TypeError("quantize_many takes tensors of one dtype, float32 or bfloat16")
    if outs is None:
        outs = [(torch.empty((w.numel() + 1) // 2, dtype=torch.uint8, device=w.device),
                 torch.empty((w.numel() + blocksize - 1) // blocksize, dtype=torch.float32, device=w.device))
                for w in ws]
    k = len(ws)
    sp = (ctypes.c_void_p * k)(*[_ptr(w) for w in ws])
    ns = (ctypes.c_int64 * k)(*[w.numel() for w in ws])
    pp = (ctypes.c_void_p * k)(*[_ptr(o[0]) for o in outs])
    ap = (ctypes.c_void_p * k)(*[_ptr(o[1]) for o in outs])
    st = _lib.load().nf4_quantize_many(sp, ns, k, NF4_BF16 if dt == torch.bfloat16 else NF4_F32, blocksize,
                                       _QUANT_TYPES[quant_type], pp, ap, _stream(stream))
    _lib.check(st, "nf4_quantize_many")
    return outs


def double_quant(absmax: torch.Tensor, code: str = "e4m3", dq_blocksize: int = DQ_BLOCKSIZE, out=None,
                 workspace: Optional[torch.Tensor] = None, stream=None):
    """Second-level quantization of the fp32 absmax array.
    Returns (q uint8 [nb], scale fp32 [ceil(nb/256)], mean fp32 [1])."""
    _need_cuda(absmax, "absmax")
    lib = _lib.load()
    nb = absmax.numel()
    if out is None:
        q = torch.empty(nb, dtype=torch.uint8, device=absmax.device)
        scale = torch.empty((nb + dq_blocksize - 1) // dq_blocksize, dtype=torch.float32, device=absmax.device)
        mean = torch.empty(1, dtype=torch.float32, device=absmax.device)
    else:
        q, scale, mean = out
    ws_bytes = lib.nf4_double_quant_workspace_bytes(nb)
    if workspace is None:  # a fresh zeroed buffer (a caller's own buffer is zeroed once and reused)
        workspace = torch.zeros(ws_bytes, dtype=torch.uint8, device=absmax.device)
    st = lib.nf4_double_quant(_ptr(absmax), nb, dq_blocksize, _DQ_CODES[code], _ptr(q), _ptr(scale), _ptr(mean),
                              _ptr(workspace), workspace.numel(), _stream(stream))
    _lib.check(st, "nf4_double_quant")
    return q, scale, mean


def double_quant_many(absmaxes, code: str = "e4m3", dq_blocksize: int = DQ_BLOCKSIZE, outs=None,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> list:
    """double_quant of up to 256 fp32 absmax arrays (each with its own mean) in two launches.
    Returns [(q, scale, mean)] per array, the same values double_quant gives each one."""
    absmaxes = list(absmaxes)
    if not absmaxes:
        raise ValueError("double_quant_many takes at least one array")
    lib = _lib.load()
    for a in absmaxes:
        _need_cuda(a, "absmax")
    if outs is None:
        outs = [(torch.empty(a.numel(), dtype=torch.uint8, device=a.device),
                 torch.empty((a.numel() + dq_blocksize - 1) // dq_blocksize, dtype=torch.float32, device=a.device),
                 torch.empty(1, dtype=torch.float32, device=a.device)) for a in absmaxes]
    n = len(absmaxes)
    ws_bytes = lib.nf4_double_quant_many_workspace_bytes(n)
    if workspace is None:  # a fresh zeroed buffer (a caller's own buffer is zeroed once and reused)
        workspace = torch.zeros(max(ws_bytes, 1), dtype=torch.uint8, device=absmaxes[0].device)
    ap = (ctypes.c_void_p * n)(*[_ptr(a) for a in absmaxes])
    nb = (ctypes.c_int64 * n)(*[a.numel() for a in absmaxes])
    qp = (ctypes.c_void_p * n)(*[_ptr(o[0]) for o in outs])
    sp = (ctypes.c_void_p * n)(*[_ptr(o[1]) for o in outs])
    mp = (ctypes.c_void_p * n)(*[_ptr(o[2]) for o in outs])
    st = lib.nf4_double_quant_many(ap, nb, n, dq_blocksize, _DQ_CODES[code], qp, sp, mp, _ptr(workspace),
                                   workspace.numel(), _stream(stream))
    _lib.check(st, "nf4_double_quant_many")
    return outs


def quantize_weight(w: torch.Tensor, use_double_quant: bool = True, code: str = "e4m3",
                    stream=None, quant_type: str = "nf4", blocksize: int = BLOCKSIZE) -> QuantizedWeight:
    """Quantize a 2-D weight [rows, cols] (nn.Linear layout: out x in) to NF4 (or FP4: quant_type="fp4").

    blocksize is 32, 64, 128 or 256; the matmuls take 64-element blocks only (dequantize takes all four)."""
    if w.dim() != 2:
        raise ValueError("quantize_weight takes a 2-D [rows, cols] tensor")
    packed, absmax = quantize(w, blocksize=blocksize, stream=stream, quant_type=quant_type)
    qt = _QUANT_TYPES[quant_type]
    qw = QuantizedWeight(packed=packed, rows=w.shape[0], cols=w.shape[1], absmax=absmax, blocksize=blocksize,
                         quant_type=qt)
    if use_double_quant:
        q, scale, mean = double_quant(absmax, code, stream=stream)
        qw = QuantizedWeight(packed=packed, rows=w.shape[0], cols=w.shape[1], absmax_q=q, absmax_scale=scale,
                             absmax_mean=mean, dq_code=_DQ_CODES[code], blocksize=blocksize, quant_type=qt)
    return qw


def dequantize(qw: QuantizedWeight, dtype: torch.dtype = torch.float32, out=None, stream=None) -> torch.Tensor:
    """Expand to fp32 or bf16 [rows, cols]."""
    if dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("dequantize produces float32 or bfloat16")
    if out is None:
        out = torch.empty(qw.rows, qw.cols, dtype=dtype, device=qw.packed.device)
    d = qw.descriptor()
    st = _lib.load().nf4_dequantize(ctypes.byref(d), _ptr(out), NF4_BF16 if dtype == torch.bfloat16 else NF4_F32,
                                    _stream(stream))
    _lib.check(st, "nf4_dequantize")
    return out


def gemv(qw: QuantizedWeight, x: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """y[b, n] = bf16(sum_k Wc[n, k] x[b, k]) for x bf16 [B, cols], 1 <= B <= 8."""
    _need_cuda(x, "x")
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    x2 = x.reshape(-1, qw.cols)
    if out is None:
        out = torch.empty(x2.shape[0], qw.rows, dtype=torch.bfloat16, device=x.device)
    d = qw.descriptor()
    st = _lib.load().nf4_gemv(ctypes.byref(d), _ptr(x2), x2.shape[0], _ptr(out), _stream(stream))
    _lib.check(st, "nf4_gemv")
    return out


def gemv_grouped(qws, x: torch.Tensor, outs=None, stream=None) -> list:
    """nf4_gemv of up to 4 weights with the same cols on one input x (bf16 [B, cols], B <= 8), in one launch."""
    _need_cuda(x, "x")
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    qws = list(qws)
    cols = qws[0].cols
    x2 = x.reshape(-1, cols)
    if outs is None:
        outs = [torch.empty(x2.shape[0], q.rows, dtype=torch.bfloat16, device=x.device) for q in qws]
    ds = [q.descriptor() for q in qws]
    arr = (ctypes.POINTER(_lib.NF4Weight) * len(ds))(*[ctypes.pointer(d) for d in ds])
    ys = (ctypes.c_void_p * len(outs))(*[_ptr(o) for o in outs])
    st = _lib.load().nf4_gemv_grouped(arr, len(ds), _ptr(x2), x2.shape[0], ys, _stream(stream))
    _lib.check(st, "nf4_gemv_grouped")
    return outs


GEMV_STREAM_MAX = 256


def gemv_stream(qws, xs, outs=None, stream=None) -> list:
    """nf4_gemv of up to 256 weights, each on its own input xs[i] (bf16 [B, cols_i], the same B <= 8 for all),
    in one launch.  Returns the outputs (bf16 [B, rows_i])."""
    qws, xs = list(qws), list(xs)
    if len(qws) != len(xs) or not qws:
        raise ValueError("gemv_stream takes one input per weight")
    x2 = []
    for q, x in zip(qws, xs):
        _need_cuda(x, "x")
        if x.dtype != torch.bfloat16:
            raise TypeError("x must be bfloat16")
        x2.append(x.reshape(-1, q.cols))
    batch = x2[0].shape[0]
    if any(x.shape[0] != batch for x in x2):
        raise ValueError("every input needs the same batch")
    if outs is None:
        outs = [torch.empty(batch, q.rows, dtype=torch.bfloat16, device=x2[0].device) for q in qws]
    ds = (_lib.NF4Weight * len(qws))(*[q.descriptor() for q in qws])
    xp = (ctypes.c_void_p * len(x2))(*[_ptr(x) for x in x2])
    yp = (ctypes.c_void_p * len(outs))(*[_ptr(o) for o in outs])
    st = _lib.load().nf4_gemv_stream(ds, xp, yp, len(qws), batch, _stream(stream))
    _lib.check(st, "nf4_gemv_stream")
    return outs


def gemm(qw: QuantizedWeight, x: torch.Tensor, out=None, workspace: Optional[torch.Tensor] = None,
         stream=None) -> torch.Tensor:
    """Y[m, n] = bf16(sum_k Wc[n, k] X[m, k]) for X bf16 [M, cols]."""
    _need_cuda(x, "x")
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    x2 = x.reshape(-1, qw.cols)
    m = x2.shape[0]
    lib = _lib.load()
    d = qw.descriptor()
    if out is None:
        out = torch.empty(m, qw.rows, dtype=torch.bfloat16, device=x.device)
    ws_bytes = lib.nf4_gemm_workspace_bytes(ctypes.byref(d), m)
    if workspace is None and ws_bytes:
        workspace = torch.zeros(ws_bytes, dtype=torch.uint8, device=x.device)  # zeroed once, then reusable
    st = lib.nf4_gemm(ctypes.byref(d), _ptr(x2), m, _ptr(out), _ptr(workspace),
                      workspace.numel() if workspace is not None else 0, _stream(stream))
    _lib.check(st, "nf4_gemm")
    return out


def gemm_workspace_bytes(qw: QuantizedWeight, m: int) -> int:
    """Scratch bytes nf4_gemm needs for `m` activation rows (0 when none)."""
    d = qw.descriptor()
    return int(_lib.load().nf4_gemm_workspace_bytes(ctypes.byref(d), m))


def gemm_lora(qw: QuantizedWeight, x: torch.Tensor, down: torch.Tensor, up: torch.Tensor, scale: float,
              out=None, workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Y = bf16(X . Wc^T + scale * (X . down^T) . up^T): the 4-bit matmul with a low-rank adapter
    (down bf16 [r, cols], up bf16 [rows, r], r in {16, 32}); the adapter's intermediate is not rounded."""
    for t, name in ((x, "x"), (down, "down"), (up, "up")):
        _need_cuda(t, name)
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16")
    r = down.shape[0]
    if down.shape != (r, qw.cols) or up.shape != (qw.rows, r) or not down.is_contiguous() or not up.is_contiguous():
        raise ValueError("down must be [r, cols] and up [rows, r], contiguous")
    x2 = x.reshape(-1, qw.cols)
    m = x2.shape[0]
    lib = _lib.load()
    d = qw.descriptor()
    if out is None:
        out = torch.empty(m, qw.rows, dtype=torch.bfloat16, device=x.device)
    ws_bytes = lib.nf4_gemm_lora_workspace_bytes(ctypes.byref(d), m)
    if workspace is None:
        workspace = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=x.device)  # zeroed once, then reusable
    lo = _lib.NF4Lora(_ptr(down), _ptr(up), r, float(scale))
    st = lib.nf4_gemm_lora(ctypes.byref(d), ctypes.byref(lo), _ptr(x2), m, _ptr(out), _ptr(workspace),
                           workspace.numel(), _stream(stream))
    _lib.check(st, "nf4_gemm_lora")
    return out


def gemm_lora_workspace_bytes(qw: QuantizedWeight, m: int) -> int:
    """Scratch bytes nf4_gemm_lora needs for `m` activation rows."""
    d = qw.descriptor()
    return int(_lib.load().nf4_gemm_lora_workspace_bytes(ctypes.byref(d), m))


def gemm_dx(qw: QuantizedWeight, dy: torch.Tensor, out=None, workspace: Optional[torch.Tensor] = None,
            stream=None) -> torch.Tensor:
    """Input gradient of ``gemm``: dX[m, k] = bf16(sum_n dY[m, n] Wc[n, k]) for dY bf16 [M, rows]."""
    _need_cuda(dy, "dy")
    if dy.dtype != torch.bfloat16:
        raise TypeError("dy must be bfloat16")
    dy2 = dy.reshape(-1, qw.rows)
    m = dy2.shape[0]
    lib = _lib.load()
    d = qw.descriptor()
    if out is None:
        out = torch.empty(m, qw.cols, dtype=torch.bfloat16, device=dy.device)
    ws_bytes = lib.nf4_gemm_dx_workspace_bytes(ctypes.byref(d), m)
    if workspace is None and ws_bytes:
        workspace = torch.zeros(ws_bytes, dtype=torch.uint8, device=dy.device)  # zeroed once, then reusable
    st = lib.nf4_gemm_dx(ctypes.byref(d), _ptr(dy2), m, _ptr(out), _ptr(workspace),
                         workspace.numel() if workspace is not None else 0, _stream(stream))
    _lib.check(st, "nf4_gemm_dx")
    return out


def gemm_dx_workspace_bytes(qw: QuantizedWeight, m: int) -> int:
    """Scratch bytes nf4_gemm_dx needs for `m` gradient rows (0 when none)."""
    d = qw.descriptor()
    return int(_lib.load().nf4_gemm_dx_workspace_bytes(ctypes.byref(d), m))


def storage_bytes(n: int, use_double_quant: bool = True) -> int:
    return int(_lib.load().nf4_storage_bytes(n, BLOCKSIZE, 1 if use_double_quant else 0, DQ_BLOCKSIZE))


def code_table() -> list:
    buf = (ctypes.c_float * 16)()
    _lib.load().nf4_code_table(buf)
    return list(buf)


def kernel_launches() -> int:
    """Kernels launched through the library by this process so far."""
    return int(_lib.load().nf4_kernel_launches())


def check_device_error(stream=None) -> None:
    _lib.check(_lib.load().nf4_check_device_error(_stream(stream)), "device error word")
