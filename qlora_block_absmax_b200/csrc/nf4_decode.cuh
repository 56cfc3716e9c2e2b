// nf4_decode.cuh -- register decode of packed NF4 codes into bf16 pairs.
//
// "bitsandbytes" (ozercemkelahmet.com/tools), "How it works" Step 5: a block is
// expanded back to 16-bit with its scale and the code book.  For one level-1
// block with scale a, the 16 possible 16-bit weights are bf16_rn(RN(code[i] * a))
// ("bitsandbytes quantization tutorial", mljourney.com: compute dtype bfloat16).
// They are built once per block and kept as byte-permute pools: the low and the
// high byte of entries 0..7 and of entries 8..15, 8 bytes each.  A packed word
// of 8 codes is then decoded with byte permutes: each code nibble is a permute
// selector, and bit 3 of the nibble (which pool half) picks between two
// lookups through a byte mask.
#pragma once
#include "nf4_common.cuh"

namespace nf4 {

struct Table {  // byte pools: low/high bytes of bf16(code[i] * a), i in 0..7 (A) and 8..15 (B)
  uint32_t la0, la1, lb0, lb1, ha0, ha1, hb0, hb1;
};

// kBook: the code book, 0 = NF4, 1 = FP4 (E2M1 / 6 by bit pattern; "bitsandbytes", "Glossary")
template <int kBook = 0>
__device__ __forceinline__ Table make_table(float a) {
  constexpr float nf4[16] = NF4_CODE_INIT;
  constexpr float fp4[16] = FP4_CODE_INIT;
  uint32_t r[8];
#pragma unroll
  for (int m = 0; m < 8; ++m)
    r[m] = pack_bf16x2(__fmul_rn(kBook ? fp4[2 * m] : nf4[2 * m], a),
                       __fmul_rn(kBook ? fp4[2 * m + 1] : nf4[2 * m + 1], a));
  Table T;
  T.la0 = prmt(r[0], r[1], 0x6420);
  T.la1 = prmt(r[2], r[3], 0x6420);
  T.lb0 = prmt(r[4], r[5], 0x6420);
  T.lb1 = prmt(r[6], r[7], 0x6420);
  T.ha0 = prmt(r[0], r[1], 0x7531);
  T.ha1 = prmt(r[2], r[3], 0x7531);
  T.hb0 = prmt(r[4], r[5], 0x7531);
  T.hb1 = prmt(r[6], r[7], 0x7531);
  return T;
}

// Multipliers the decode reads at run time (65536 and 255).  Because the
// compiler cannot see their values, `q * 65536 >> 32` and `m * 255` stay
// integer multiplies, which run on the FMA pipe; the shift and the logic op
// they replace would compete with the byte permutes for the ALU pipe.
namespace {
__constant__ uint32_t c_decode_mul[2] = {65536u, 255u};
}
struct DecodeMul {
  uint32_t hi16, ff;
};
__device__ __forceinline__ DecodeMul decode_mul() { return DecodeMul{c_decode_mul[0], c_decode_mul[1]}; }

// Decode 8 codes (one packed word) into 4 bf16x2 registers:
// out[0] = (e0, e1), out[1] = (e2, e3), out[2] = (e4, e5), out[3] = (e6, e7),
// element e_j being the j-th code in memory order (high nibble first).
__device__ __forceinline__ void decode_word(uint32_t q, const Table& T, uint32_t (&out)[4], const DecodeMul& k) {
  const uint32_t qx = q ^ 0x88888888u;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t s = h ? __umulhi(q, k.hi16) : q;    // 4 selector nibbles
    const uint32_t sx = h ? __umulhi(qx, k.hi16) : qx; // same, pool-B view (bit 3 flipped)
    const uint32_t la = prmt(T.la0, T.la1, s), lb = prmt(T.lb0, T.lb1, sx);
    const uint32_t ha = prmt(T.ha0, T.ha1, s), hb = prmt(T.hb0, T.hb1, sx);
    // 0x01 where code >= 8 (plain selector), 0x00 where code < 8 (sign mode of a byte whose top bit is 0)
    const uint32_t m1 = prmt(0x01010101u, 0x01010101u, sx);
    const uint32_t M = m1 * k.ff;                               // 0xff where code >= 8
    const uint32_t L = (la & ~M) | (lb & M);
    const uint32_t H = (ha & ~M) | (hb & M);
    out[2 * h] = prmt(L, H, 0x4051);      // selector nibble k -> element: 1,0,3,2
    out[2 * h + 1] = prmt(L, H, 0x6273);
  }
}

// Same with compile-time constants (the compiler picks shifts and logic ops).
__device__ __forceinline__ void decode_word(uint32_t q, const Table& T, uint32_t (&out)[4]) {
  decode_word(q, T, out, DecodeMul{65536u, 255u});
}

}  // namespace nf4
