// exact_sum.cuh -- the exact sum of fp32 values behind the double-quantization
// mean (used by the double-quant sum kernel).
//
// "bitsandbytes" (ozercemkelahmet.com/tools), "Double quantization": the
// level-1 scales are centred by their mean before the second quantization.
// The mean is mu = fp32(fp64(exact sum) / nb): every fp32 value is an integer
// multiple of 2^-149, so the sum is exact in a 320-bit fixed-point number held
// as ten signed 64-bit limbs of 32-bit digits; integer addition makes it
// independent of order.
#pragma once
#include "nf4_common.cuh"

namespace nf4 {
namespace {

constexpr int kLimbs = 10;

struct SumWorkspace {
  unsigned long long limb[kLimbs];  // two's-complement running sums of 32-bit digits
  unsigned int count;               // CTAs of the running sum that have added their share
};

// An fp32 value x is +-mant * 2^(sh - 149) with mant < 2^24 and 0 <= sh <= 253: the
// 56-bit chunk mant << (sh mod 32) placed at limb sh / 32.
struct Chunk {
  long long v;  // signed chunk, |v| < 2^56
  int li;       // limb of its lowest bit
};
__device__ __forceinline__ Chunk chunk_of(float x) {
  const uint32_t u = __float_as_uint(x);
  const uint32_t e = (u >> 23) & 0xffu, f = u & 0x7fffffu;
  const uint32_t mant = e ? (f | 0x800000u) : f;
  const int sh = e ? (int)e - 1 : 0;
  const long long v = (long long)((uint64_t)mant << (sh & 31));
  return Chunk{(u >> 31) ? -v : v, sh >> 5};
}

// Per-thread running sum: chunks at limb `base` and `base + 1` add into two 64-bit
// registers (exact while fewer than 2^7 chunks have been added); any other limb, and
// every 64 values, goes to the CTA's shared limbs as balanced 32-bit digits
// (|digit| <= 2^31, so no limb total over 2^31 values leaves the signed 64-bit range).
struct Runner {
  int base = -1;
  long long a0 = 0, a1 = 0;
  int n = 0;
};

__device__ __forceinline__ void shared_add(long long* limbs, int li, long long v) {
  atomicAdd(reinterpret_cast<unsigned long long*>(limbs + li), (unsigned long long)v);  // wraps: signed add
}

// the low 32 bits of v as a signed digit in [-2^31, 2^31): v - low(v) is a multiple of 2^32
__device__ __forceinline__ long long low_digit(long long v) { return (long long)(int32_t)(uint32_t)v; }

// digits of a0 (at base) and a1 (at base + 1): a = lo + 2^32 hi with balanced lo
__device__ __forceinline__ void runner_digits(const Runner& r, long long& d0, long long& d1, long long& d2) {
  const long long l0 = low_digit(r.a0), l1 = low_digit(r.a1);
  d0 = l0;
  d1 = ((r.a0 - l0) >> 32) + l1;
  d2 = (r.a1 - l1) >> 32;
}

__device__ __forceinline__ void runner_flush(Runner& r, long long* limbs) {
  if (r.base < 0) return;
  long long d0, d1, d2;
  runner_digits(r, d0, d1, d2);
  if (d0) shared_add(limbs, r.base, d0);
  if (d1) shared_add(limbs, r.base + 1, d1);
  if (d2) shared_add(limbs, r.base + 2, d2);
  r.a0 = r.a1 = 0;
  r.n = 0;
}

__device__ __forceinline__ void runner_add(Runner& r, float x, long long* limbs) {
  const Chunk c = chunk_of(x);
  if (r.base < 0) r.base = c.li;
  if (c.li == r.base) {
    r.a0 += c.v;
  } else if (c.li == r.base + 1) {
    r.a1 += c.v;
  } else {  // rare: a value more than 2^32 away in magnitude from this thread's first
    const long long lo = low_digit(c.v);
    shared_add(limbs, c.li, lo);
    shared_add(limbs, c.li + 1, (c.v - lo) >> 32);
  }
  if (++r.n == 64) runner_flush(r, limbs);
}

// limb i of d (0 <= i < kLimbs), else 0; unrolled so d stays in registers
__device__ __forceinline__ uint32_t limb_at(const uint32_t (&d)[kLimbs], int i) {
  uint32_t v = 0;
#pragma unroll
  for (int L = 0; L < kLimbs; ++L) v = (L == i) ? d[L] : v;
  return v;
}

// bits [pos, pos + 64) of the 320-bit number d (pos may be negative)
__device__ __forceinline__ uint64_t window64(const uint32_t (&d)[kLimbs], int pos) {
  const int i = pos >> 5;  // floor division
  const int s = pos & 31;
  const uint32_t l0 = limb_at(d, i), l1 = limb_at(d, i + 1), l2 = limb_at(d, i + 2);
  const uint64_t lo = ((uint64_t)l1 << 32) | l0;
  if (s == 0) return lo;
  return (lo >> s) | ((uint64_t)l2 << (64 - s));
}

// Normalise the signed limbs, round the total to fp64 (nearest even) and
// return mu = fp32(fp64 sum / nb).  Single thread, registers only.
__device__ float finish_mean(const long long (&limb_in)[kLimbs], int64_t nb) {
  long long l[kLimbs];
#pragma unroll
  for (int L = 0; L < kLimbs; ++L) l[L] = limb_in[L];
#pragma unroll
  for (int L = 0; L < kLimbs - 1; ++L) {  // carry: limbs 0..8 into [0, 2^32)
    const long long carry = l[L] >> 32;   // arithmetic shift = floor division
    l[L] -= carry * (1LL << 32);
    l[L + 1] += carry;
  }
  const bool neg = l[kLimbs - 1] < 0;
  uint32_t d[kLimbs];
  if (neg) {  // magnitude of a negative total: subtract from zero
    long long borrow = 0;
#pragma unroll
    for (int L = 0; L < kLimbs - 1; ++L) {
      const long long t = -l[L] - borrow;
      borrow = t < 0;
      d[L] = (uint32_t)(t + (borrow ? (1LL << 32) : 0));
    }
    d[kLimbs - 1] = (uint32_t)(-l[kLimbs - 1] - borrow);
  } else {
#pragma unroll
    for (int L = 0; L < kLimbs; ++L) d[L] = (uint32_t)l[L];
  }
  int top = -1;  // index of the highest set bit
#pragma unroll
  for (int L = 0; L < kLimbs; ++L)
    if (d[L]) top = 32 * L + 31 - __clz(d[L]);
  double s = 0.0;
  if (top >= 0) {
    uint64_t m;
    int exp2;  // s = m * 2^exp2
    if (top < 53) {
      m = window64(d, 0);
      exp2 = -149;
    } else {
      const int low = top - 52;  // lowest kept bit
      const uint64_t w = window64(d, low - 1);  // round bit + 53 kept bits
      m = (w >> 1) & ((1ull << 53) - 1);
      const bool round = w & 1u;
      bool sticky = false;  // any set bit below low - 1
      const int sb = low - 1;
#pragma unroll
      for (int L = 0; L < kLimbs; ++L) {
        const int base = 32 * L;
        uint32_t mask = 0;
        if (base + 32 <= sb) mask = 0xffffffffu;
        else if (base < sb) mask = (1u << (sb - base)) - 1u;
        sticky |= (d[L] & mask) != 0;
      }
      if (round && (sticky || (m & 1u))) m += 1;  // may reach 2^53: still exact
      exp2 = low - 149;
    }
    // m < 2^54 and -149 <= exp2 <= 118: both factors exact, product exact
    s = __dmul_rn((double)m, __longlong_as_double((long long)(exp2 + 1023) << 52));
  }
  if (neg) s = -s;
  return __double2float_rn(__ddiv_rn(s, (double)nb));
}

// Hand a warp's runners to the CTA's shared limbs: one set of digits (three
// limbs) when every lane has the same base, the usual case; else lane by lane.
__device__ __forceinline__ void runner_warp_flush(Runner& r, long long* limbs) {
  const int wbase = __reduce_max_sync(0xffffffffu, r.base);
  if (r.base < 0) r.base = wbase;  // lanes without values hold zeros
  if (__all_sync(0xffffffffu, r.base == wbase)) {
    long long d[3];
    runner_digits(r, d[0], d[1], d[2]);
#pragma unroll
    for (int k = 0; k < 3; ++k)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) d[k] += __shfl_xor_sync(0xffffffffu, d[k], off);
    if ((threadIdx.x & 31) == 0 && wbase >= 0)
#pragma unroll
      for (int k = 0; k < 3; ++k)
        if (d[k]) shared_add(limbs, wbase + k, d[k]);
  } else {
    runner_flush(r, limbs);
  }
  r.base = -1;
  r.a0 = r.a1 = 0;
  r.n = 0;
}

}  // namespace
}  // namespace nf4
