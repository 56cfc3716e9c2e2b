"""Generate nf4_codebook.h: the NF4 levels and the quantizer's decision tables
for the CUDA library.

Run:  python qlora_block_absmax_b200/csrc/gen_codebook.py
(the header is committed; the build checks that it is current).

NF4 definition (web pages on bitsandbytes / QLoRA: "bitsandbytes",
ozercemkelahmet.com/tools, section "How NF4 works"; "bitsandbytes quantization
tutorial", mljourney.com, section "How NF4 Works"): the 16 levels split the
standard normal distribution into pieces of equal probability.  Read as the
QLoRA construction: normal
quantiles at equally spaced probabilities in [0.5, p*], 8 above and 7 below an
exact zero, p* = mean of (1 - 1/30) and (1 - 1/32), scaled to [-1, 1].

Quantizer decisions ("How it works", Step 3: nearest entry of the code book).
The nearest code of a normalised value x is the number of exact midpoints
(c_i + c_{i+1}) / 2 lying strictly below x (a tie goes to the lower code).  For
fp32 x the strict comparison against an exact midpoint M equals the fp32
comparison x > RD32(M), so the kernels compare against thresholds rounded
toward minus infinity.  A 32-bucket table over [-1, 1] (bucket = the low 5
mantissa bits of v = RD(16 S x + 2^23 + 16)) gives, per bucket, the count of
thresholds below it and the one threshold inside it, if any; each bucket is
held by one lane of a warp and read with a shuffle.

FP4 tables (the same scheme on magnitudes): the E2M1 values / 6 indexed by the
4-bit pattern s e1 e0 m ("bitsandbytes", "Glossary" and "What it is": FP4 is
the 4-bit floating-point format; the pages give no layout, E2M1 is read), the 7
magnitude thresholds RD32 of the exact midpoints of the positive levels (a tie
goes to the level with the even mantissa bit, which the strict comparison gives
for the one representable midpoint), and 16 buckets over [0, 1] with bucket =
the low 4 mantissa bits of RD(16 S |x| + 2^23).
"""
from __future__ import annotations

import os
import statistics
import struct
from fractions import Fraction

HERE = os.path.dirname(os.path.abspath(__file__))
OUT = os.path.join(HERE, "nf4_codebook.h")

# 32-bucket map used by the quantizer: bucket j = floor(16 * Q32_SCALE * x) + 16, i.e. x in
# [(j - 16) / (16 S), (j - 15) / (16 S)) -- the low 5 mantissa bits of RD(16 S x + 2^23 + 16)
Q32_SCALE = 1.0 - 2.0 ** -12


def f32(x: float) -> float:
    return struct.unpack("<f", struct.pack("<f", x))[0]


def f32_bits(x: float) -> int:
    return struct.unpack("<I", struct.pack("<f", x))[0]


def bits_f32(b: int) -> float:
    return struct.unpack("<f", struct.pack("<I", b & 0xFFFFFFFF))[0]


def next_down_f32(x: float) -> float:
    b = f32_bits(x)
    if x > 0:
        return bits_f32(b - 1)
    if x == 0:
        return bits_f32(0x80000001)
    return bits_f32(b + 1)


def rd32(q: Fraction) -> float:
    """largest fp32 <= q (q well inside the normal range)"""
    x = f32(float(q))
    while Fraction(x) > q:
        x = next_down_f32(x)
    return x


def levels() -> list[float]:
    nd = statistics.NormalDist()
    pstar = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0))
    neg = [-nd.inv_cdf(0.5 + (pstar - 0.5) * (k / 7.0)) for k in range(7, 0, -1)]
    pos = [nd.inv_cdf(0.5 + (pstar - 0.5) * (k / 8.0)) for k in range(1, 9)]
    v = neg + [0.0] + pos
    top = max(abs(t) for t in v)
    return [f32(t / top) for t in v]


def hexf(x: float) -> str:
    if x == 0:
        return "-0.0f" if struct.pack("<f", x)[3] & 0x80 else "0.0f"
    return float(x).hex() + "f"


def fp4_levels() -> list[float]:
    """E2M1 values / 6 by bit pattern s e1 e0 m (bias 1; e = 0 is subnormal: 0 or 0.5)"""
    out = []
    for nib in range(16):
        s, e, m = nib >> 3, (nib >> 1) & 3, nib & 1
        mag = 0.5 * m if e == 0 else (1.0 + 0.5 * m) * 2.0 ** (e - 1)
        out.append(f32((-mag if s else mag) / 6.0))
    return out


def bucket_table(thr: list[float], edge, nbuckets: int) -> list[int]:
    """entry j: bits of the one threshold inside bucket j (2.0f if none), low 4 mantissa bits = #thresholds below"""
    out = []
    for j in range(nbuckets):
        lo, hi = edge(j), edge(j + 1)
        below = sum(1 for t in thr if Fraction(t) < lo)
        ins = [t for t in thr if lo <= Fraction(t) < hi]
        assert len(ins) <= 1
        for t in ins:
            assert Fraction(t) - lo >= Fraction(1, 2 ** 19) and hi - Fraction(t) >= Fraction(1, 2 ** 19)
        t = ins[0] if ins else 2.0
        out.append((f32_bits(t) & ~15) | below)
    return out


def main() -> None:
    c = levels()
    assert len(c) == 16 and c[0] == -1.0 and c[15] == 1.0 and c[7] == 0.0
    assert all(c[i] < c[i + 1] for i in range(15))
    mids = [(Fraction(c[i]) + Fraction(c[i + 1])) / 2 for i in range(15)]
    thr = [rd32(m) for m in mids]

    # 32-bucket table: bucket j holds x in [(j - 16) / (16 S), (j - 15) / (16 S));
    # entry = bits of the threshold inside the bucket (2.0f if none) with its low
    # 4 mantissa bits replaced by the bucket's base count (the kernel resolves any
    # value within 2^-19 of an entry with the exact quotient and kThreshold[base])
    def edge32(j: int) -> Fraction:
        return (Fraction(2) + Fraction(j, 16) - 3) / Fraction(Q32_SCALE)

    q32 = bucket_table(thr, edge32, 32)
    assert edge32(0) < -1 - Fraction(1, 2 ** 20) and edge32(32) > 1 + Fraction(1, 2 ** 20)

    # FP4: magnitude thresholds between the positive levels (patterns 0..7 ascend), 16 buckets over [0, 1]
    f4 = fp4_levels()
    assert [abs(v) for v in f4[8:]] == f4[:8] and all(f4[i] < f4[i + 1] for i in range(7))
    f4mids = [(Fraction(f4[i]) + Fraction(f4[i + 1])) / 2 for i in range(7)]
    f4thr = [rd32(m) for m in f4mids]
    for i, m in enumerate(f4mids):  # an exact fp32 midpoint is a tie: the strict test keeps level i, so it must be even
        if Fraction(f4thr[i]) == m:
            assert i % 2 == 0

    def edge16(j: int) -> Fraction:
        return Fraction(j, 16) / Fraction(Q32_SCALE)

    q16 = bucket_table(f4thr, edge16, 16)
    assert edge16(16) > 1 + Fraction(1, 2 ** 20)
    lines = []
    lines.append("// Generated by gen_codebook.py -- do not edit.")
    lines.append("// NF4 code book (ascending; index 7 is exact zero) and quantizer decision tables,")
    lines.append("// as initializer lists so host and device code can both declare arrays from them.")
    lines.append("#pragma once")
    lines.append("#define NF4_CODE_INIT {" + ", ".join(hexf(x) for x in c) + "}")
    lines.append("// RD32((code[i] + code[i+1]) / 2): the code of x is #{i : x > threshold[i]}")
    lines.append("#define NF4_THRESHOLD_INIT {" + ", ".join(hexf(x) for x in thr) + "}")
    lines.append(f"#define NF4_Q32_SCALE {hexf(f32(Q32_SCALE))}")
    lines.append("// 32 quantizer buckets: threshold bits with the base count in the low 4 mantissa bits")
    lines.append("#define NF4_Q32_INIT {" + ", ".join(f"0x{b:08x}u" for b in q32) + "}")
    lines.append("// FP4 (E2M1 / 6) by bit pattern s e1 e0 m; magnitude thresholds RD32 of the positive midpoints;")
    lines.append("// 16 magnitude buckets (low 4 mantissa bits of RD(16 S |x| + 2^23)), entries as above")
    lines.append("#define FP4_CODE_INIT {" + ", ".join(hexf(x) for x in f4) + "}")
    lines.append("#define FP4_THRESHOLD_INIT {" + ", ".join(hexf(x) for x in f4thr) + "}")
    lines.append("#define FP4_Q16_INIT {" + ", ".join(f"0x{b:08x}u" for b in q16) + "}")
    text = "\n".join(lines) + "\n"
    with open(OUT, "w") as f:
        f.write(text)


def current() -> bool:
    """True when the committed header matches what this script would write."""
    import tempfile
    global OUT
    keep = OUT
    with tempfile.TemporaryDirectory() as d:
        OUT = os.path.join(d, "h")
        main()
        fresh = open(OUT).read()
    OUT = keep
    return os.path.exists(OUT) and open(OUT).read() == fresh


if __name__ == "__main__":
    main()
