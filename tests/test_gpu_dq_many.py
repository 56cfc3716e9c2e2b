"""nf4_double_quant_many against the oracle: every array's codes, second-level scales and mean bit for bit, with
arrays of every size class (1 value, short 256-blocks, arrays cut between many CTAs of the sum kernel), an empty
array among them, both 8-bit codes, arrays that sit at 16-byte offsets inside one buffer, 256 arrays in one call,
and one workspace reused across calls."""
import numpy as np
import pytest
import torch

import oracle
import qlora_block_absmax_b200 as nf4
from qlora_block_absmax_b200 import synth

pytestmark = pytest.mark.gpu

CODES = {"e4m3": oracle.DQ_E4M3, "int8": oracle.DQ_INT8}


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def arrays():
    r = synth.rng(4242)
    _, a2 = oracle.quantize(synth.bf16_4096x4096_outlier_weight().reshape(-1))
    return [
        np.abs(r.standard_normal(1)).astype(np.float32),
        (np.abs(r.standard_normal(3_000_001)) * np.exp(r.uniform(-30, 30, 3_000_001))).astype(np.float32),
        np.full(700, 0.0625, np.float32),
        np.zeros(0, np.float32),
        a2,
        r.standard_normal(257).astype(np.float32),
        np.concatenate([np.zeros(300, np.float32), np.full(212, 1e-40, np.float32)]),
        (np.abs(r.standard_normal(5)) * 1e30).astype(np.float32),
        np.abs(r.standard_normal(65536)).astype(np.float32),
        np.abs(r.standard_normal(255)).astype(np.float32),
    ]


def check(a, got, code, what):
    q, s, m = got
    q_ref, s_ref, m_ref = oracle.double_quant(a, 256, CODES[code])
    assert np.float32(m.item()).view(np.uint32) == np.float32(m_ref).view(np.uint32), what
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32)), what
    assert np.array_equal(q.cpu().numpy(), q_ref), what


@pytest.mark.parametrize("code", ["e4m3", "int8"])
def test_double_quant_many_bit_exact(code):
    arrs = arrays()
    outs = nf4.double_quant_many([dev(a) for a in arrs], code)
    nf4.check_device_error()
    for i, (a, o) in enumerate(zip(arrs, outs)):
        if a.size:
            check(a, o, code, f"array {i} ({a.size} values)")


def test_double_quant_many_matches_single_calls_and_reuses_workspace():
    """the same workspace (zeroed once) for three calls in a row: each call's results equal nf4_double_quant's,
    and the workspace is all zero again afterwards"""
    arrs = [a for a in arrays() if a.size]
    ws = torch.zeros(nf4._lib.load().nf4_double_quant_many_workspace_bytes(len(arrs)), dtype=torch.uint8,
                     device="cuda")
    for code in ("e4m3", "int8", "e4m3"):
        outs = nf4.double_quant_many([dev(a) for a in arrs], code, workspace=ws)
        for a, (q, s, m) in zip(arrs, outs):
            q1, s1, m1 = nf4.double_quant(dev(a), code)
            assert torch.equal(q, q1) and torch.equal(s.view(torch.int32), s1.view(torch.int32))
            assert torch.equal(m.view(torch.int32), m1.view(torch.int32))
    torch.cuda.synchronize()
    assert int(ws.count_nonzero()) == 0
    nf4.check_device_error()


def test_double_quant_many_views_of_one_buffer():
    """arrays that are 16-byte aligned slices of one buffer, outputs likewise"""
    r = synth.rng(77)
    sizes = [4, 256, 1, 1028, 512, 8, 3000]
    offs = np.cumsum([0] + [(n + 3) // 4 * 4 for n in sizes])
    whole = (np.abs(r.standard_normal(int(offs[-1]))) + 0.01).astype(np.float32)
    buf = dev(whole)
    qbuf = torch.empty(int(offs[-1]) + 16 * len(sizes), dtype=torch.uint8, device="cuda")
    views, outs, qoff = [], [], 0
    for n, o in zip(sizes, offs[:-1]):
        views.append(buf[int(o):int(o) + n])
        outs.append((qbuf[qoff:qoff + n], torch.empty((n + 255) // 256, dtype=torch.float32, device="cuda"),
                     torch.empty(1, dtype=torch.float32, device="cuda")))
        qoff += (n + 15) // 16 * 16
    nf4.double_quant_many(views, "e4m3", outs=outs)
    nf4.check_device_error()
    for i, (n, o) in enumerate(zip(sizes, offs[:-1])):
        check(whole[int(o):int(o) + n], outs[i], "e4m3", f"view {i}")


def test_double_quant_many_256_arrays():
    r = synth.rng(5150)
    sizes = r.integers(1, 3000, 256)
    arrs = [(np.abs(r.standard_normal(int(n))) * np.exp(r.uniform(-5, 5, int(n)))).astype(np.float32) for n in sizes]
    outs = nf4.double_quant_many([dev(a) for a in arrs], "e4m3")
    nf4.check_device_error()
    for i, (a, o) in enumerate(zip(arrs, outs)):
        check(a, o, "e4m3", f"array {i}")
