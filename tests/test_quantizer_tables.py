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
    if s in ("0.0", "-0.0"):
        return -0.0 if s.startswith("-") else 0.0
    return float.fromhex(s)


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


def test_fp4_tables_match_the_oracle_and_decide_every_magnitude():
    """FP4 tables: the levels are the oracle's E2M1 / 6 by pattern (signed zero included); the magnitude
    thresholds are the largest fp32 values not above the exact midpoints; the 16-bucket rule on |q| gives the
    threshold count for every fp32 magnitude in [0, 1] it trusts; and sign + count is the oracle's nearest code"""
    _, f4 = oracle.fp4_codebook()
    code = np.array([_hexf(s) for s in _init("FP4_CODE_INIT")], np.float32)
    assert np.array_equal(code.view(np.uint32), f4.view(np.uint32))  # bit for bit, -0 at pattern 8
    thr = np.array([_hexf(s) for s in _init("FP4_THRESHOLD_INIT")], np.float32)
    for i in range(7):
        mid = (Fraction(float(f4[i])) + Fraction(float(f4[i + 1]))) / 2
        assert Fraction(float(thr[i])) <= mid < Fraction(float(np.nextafter(thr[i], np.float32(2))))
    q16 = np.array([int(s.rstrip("u"), 16) for s in _init("FP4_Q16_INIT")], np.uint32)
    scale16 = np.float32(16.0) * np.float32(_hexf(_init_scalar("NF4_Q32_SCALE")))
    e_thr = q16.view(np.float32)
    near = np.float32(2.0 ** -19)
    top = int(np.float32(1.0).view(np.uint32)) + 1
    checked = 0
    for lo in range(0, top, 1 << 24):
        q = np.arange(lo, min(lo + (1 << 24), top), dtype=np.uint32).view(np.float32)
        bucket = np.floor(q.astype(np.float64) * np.float64(scale16)).astype(np.int64) & 15  # RD(16 S q + 2^23)
        e = q16[bucket]
        t = e_thr[bucket]
        fast = (e & 15).astype(np.int64) + (q > t)
        truth = np.searchsorted(thr, q, side="left")
        trusted = np.abs(q - t) > near
        assert not (trusted & (fast != truth)).any()
        checked += int(trusted.sum())
    assert checked > 1_000_000_000
    # sign + threshold count is the oracle's nearest FP4 code (ties to even, signed zero), around every threshold
    xs = []
    for t in thr:
        v = np.float32(t)
        for k in range(-3, 4):
            w = v
            for _ in range(abs(k)):
                w = np.nextafter(w, np.float32(2.0 if k > 0 else -2.0))
            xs += [float(w), -float(w)]
    xs += [0.0, -0.0, 1.0, -1.0] + list(np.random.default_rng(5).uniform(-1, 1, 2000).astype(np.float32).astype(float))
    for x in xs:
        mag = int(np.searchsorted(thr, np.float32(abs(x)), side="left"))
        assert oracle.fp4_nearest_code(x) == (8 if np.signbit(x) else 0) | mag, x
