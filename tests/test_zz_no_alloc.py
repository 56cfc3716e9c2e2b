"""nf4_double_quant_noalloc: double quantization for callers that cannot
allocate device memory (a fixed memory budget, or a host framework that owns
the allocator), with its scratch in a static array inside the library.

Called through the C ABI and compared with nf4_double_quant (caller-provided
workspace) bit for bit -- the tolerance every double-quant test uses: two calls
in a row on the shared array, with different sizes, each match the workspace
entry point exactly.
"""
import ctypes

import numpy as np
import pytest
import torch

from qlora_block_absmax_b200 import _lib, synth

pytestmark = pytest.mark.gpu


def ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def run(lib, absmax, code, noalloc):
    nb = absmax.numel()
    q = torch.empty(nb, dtype=torch.uint8, device="cuda")
    scale = torch.empty((nb + 255) // 256, dtype=torch.float32, device="cuda")
    mean = torch.empty(1, dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if noalloc:
        st = lib.nf4_double_quant_noalloc(ptr(absmax), nb, 256, code, ptr(q), ptr(scale), ptr(mean), stream)
    else:
        ws = torch.zeros(lib.nf4_double_quant_workspace_bytes(nb), dtype=torch.uint8, device="cuda")
        st = lib.nf4_double_quant(ptr(absmax), nb, 256, code, ptr(q), ptr(scale), ptr(mean), ptr(ws),
                                  ws.numel(), stream)
    assert st == 0, _lib.STATUS_NAMES.get(st, st)
    torch.cuda.synchronize()
    return q.cpu().numpy(), scale.cpu().numpy().view(np.uint32), mean.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("code", [_lib.NF4_DQ_E4M3, _lib.NF4_DQ_INT8])
def test_noalloc_matches_workspace_entry_point_twice(code):
    lib = _lib.load()
    r = synth.rng(404)
    inputs = [torch.from_numpy(np.abs(r.standard_normal(262144)).astype(np.float32) * np.float32(0.05)).cuda(),
              torch.from_numpy(np.abs(r.standard_normal(1000 * 64 + 17)).astype(np.float32)).cuda()]
    for a in inputs:  # two calls in a row on the shared scratch
        want = run(lib, a, code, noalloc=False)
        got = run(lib, a, code, noalloc=True)
        for g, w in zip(got, want):
            assert np.array_equal(g, w)
    assert lib.nf4_check_device_error(None) == 0


def test_noalloc_rejects_counts_beyond_its_limit():
    lib = _lib.load()
    dummy = torch.empty(16, dtype=torch.float32, device="cuda")
    too_many = 2 ** 31  # one past the documented maximum
    st = lib.nf4_double_quant_noalloc(ptr(dummy), too_many, 256, 0, ptr(dummy), ptr(dummy), ptr(dummy), None)
    assert _lib.STATUS_NAMES[st] == "NF4_ERR_INVALID_ARG"
