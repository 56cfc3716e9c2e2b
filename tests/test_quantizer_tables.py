"""The quantizer's generated decision tables, checked on the CPU against the oracle's code book.

The kernel decides the code of q = fp32(w * RN(1/a)) with one round-down FMA v = RD(q * 16S + 2^23 + 16), whose low
5 mantissa bits name one of 32 buckets over [-1, 1]; each bucket's table entry is the single threshold inside it
(its low 4 mantissa bits replaced by the number of thresholds below the bucket) and the code is that count plus
(q > entry).  Values within 2^-19 of the entry are re-decided with the exact quotient.  Here the rule is run for
every fp32 value in [-1, 1] (2.1e9 of them) and must give #{i : q > threshold_i} wherever the kernel trusts it.
"""
import os
import re
from fractions import Fraction

import numpy as np

import oracle

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "qlora_block_absmax_b200", "csrc",
                      "nf4_codebook.h")


def _init(name):
    text = open(HEADER).read()
    body = re.search(r"#define " + name + r" \{([^}]*)\}", text).group(1)
    return [v.strip() for v in body.split(",")]


def _hexf(s):
    s = s.rstrip("f")
    return 0.0 if s in ("0.0", "-0.0") else float.fromhex(s)


def test_thresholds_are_rd32_of_the_oracle_midpoints():
    _, c32 = oracle.codebook()
    thr = np.array([_hexf(s) for s in _init("NF4_THRESHOLD_INIT")], np.float32)
    code = np.array([_hexf(s) for s in _init("NF4_CODE_INIT")], np.float32)
    assert np.array_equal(code, c32)
    for i in range(15):
        mid = (Fraction(float(c32[i])) + Fraction(float(c32[i + 1]))) / 2
        t = Fraction(float(thr[i]))
        assert t <= mid and Fraction(float(np.nextafter(thr[i], np.float32(2)))) > mid  # largest fp32 <= midpoint


def test_bucket_rule_decides_every_fp32_in_range():
    thr = np.array([_hexf(s) for s in _init("NF4_THRESHOLD_INIT")], np.float32)
    q32 = np.array([int(s.rstrip("u"), 16) for s in _init("NF4_Q32_INIT")], np.uint32)
    scale16 = np.float32(16.0) * np.float32(_hexf(_init_scalar("NF4_Q32_SCALE")))  # 16 S, exact in fp32
    e_thr = q32.view(np.float32)
    near = np.float32(2.0 ** -19)
    checked = 0
    step = 1 << 24
    top = int(np.float32(1.0).view(np.uint32)) + 1
    for sign in (0, 0x80000000):
        for lo in range(0, top, step):
            bits = np.arange(lo, min(lo + step, top), dtype=np.uint32) | np.uint32(sign)
            q = bits.view(np.float32)
            # RD(q * 16S + 2^23 + 16) = 2^23 + 16 + floor(q * 16S): the product is exact in fp64
            bucket = (np.floor(q.astype(np.float64) * np.float64(scale16)).astype(np.int64) + 16) & 31
            e = q32[bucket]
            t = e_thr[bucket]
            fast = (e & 15).astype(np.int64) + (q > t)
            truth = np.searchsorted(thr, q, side="left")  # #{i : threshold_i < q}
            trusted = np.abs(q - t) > near
            bad = trusted & (fast != truth)
            assert not bad.any(), f"q = {q[bad][:4]}"
            checked += int(trusted.sum())
    assert checked > 2_000_000_000


def _init_scalar(name):
    text = open(HEADER).read()
    return re.search(r"#define " + name + r" (\S+)", text).group(1)
