"""nf4_quantize_many against the oracle: every tensor's packed codes and absmax bit for bit, for bf16 and fp32
sources, every level-1 block size, both code books, sizes from 1 element to tensors that span many warp
iterations (with short last blocks and odd tails), an empty tensor among them, views into one buffer, and 256
tensors in one call; each result also equals the one-tensor call's."""
import numpy as np
import pytest
import torch

import oracle
import qlora_block_absmax_b200 as nf4
from qlora_block_absmax_b200 import synth

pytestmark = pytest.mark.gpu


def sources(dtype, seed):
    r = synth.rng(seed)
    sizes = [1, 63, 64, 65, 1000, 4096 * 17 + 3, 0, 1 << 20, 7, 256 * 33]
    out = []
    for i, n in enumerate(sizes):
        w = (r.standard_normal(n) * np.exp(r.uniform(-3, 3, n)) * 0.02).astype(np.float32)
        if n > 100:
            w[r.integers(0, n, 5)] *= 40  # a few outliers
        if i == 4:
            w[:128] = 0.0  # all-zero blocks
        out.append(synth.f32_to_bf16_bits(w) if dtype == "bf16" else w)
    return out


def dev(a: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.view(torch.bfloat16) if a.dtype == np.uint16 else t


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("blocksize", [32, 64, 128, 256])
@pytest.mark.parametrize("book", ["nf4", "fp4"])
def test_quantize_many_bit_exact(dtype, blocksize, book):
    srcs = sources(dtype, 1000 + blocksize)
    devs = [dev(s) for s in srcs]
    outs = nf4.quantize_many(devs, blocksize=blocksize, quant_type=book)
    nf4.check_device_error()
    ref_fn = oracle.quantize if book == "nf4" else oracle.fp4_quantize
    for i, (s, (p, a)) in enumerate(zip(srcs, outs)):
        if s.size == 0:
            continue
        p_ref, a_ref = ref_fn(s, blocksize)
        assert np.array_equal(p.cpu().numpy(), p_ref), (i, s.size)
        assert np.array_equal(a.cpu().numpy().view(np.uint32), a_ref.view(np.uint32)), (i, s.size)
        p1, a1 = nf4.quantize(devs[i], blocksize=blocksize, quant_type=book)
        assert torch.equal(p, p1) and torch.equal(a.view(torch.int32), a1.view(torch.int32)), (i, s.size)


def test_quantize_many_views_and_256_tensors():
    r = synth.rng(31)
    sizes = r.integers(1, 5000, 256)
    offs = np.cumsum([0] + [(int(n) + 7) // 8 * 8 for n in sizes])  # bf16 views at 16-byte offsets
    whole = synth.f32_to_bf16_bits((r.standard_normal(int(offs[-1])) * 0.02).astype(np.float32))
    buf = dev(whole)
    views = [buf[int(o):int(o) + int(n)] for n, o in zip(sizes, offs[:-1])]
    outs = nf4.quantize_many(views)
    nf4.check_device_error()
    for i, (n, o) in enumerate(zip(sizes, offs[:-1])):
        p_ref, a_ref = oracle.quantize(whole[int(o):int(o) + int(n)])
        assert np.array_equal(outs[i][0].cpu().numpy(), p_ref), i
        assert np.array_equal(outs[i][1].cpu().numpy().view(np.uint32), a_ref.view(np.uint32)), i
