// quantize.cu -- blockwise NF4 quantization (level 1).
//
// "bitsandbytes" (ozercemkelahmet.com/tools), "How it works":
//   Step 1  blocks of 64 consecutive values,
//   Step 2  the block's absmax is its scale; every value is divided by it,
//   Step 3  each scaled value takes the nearest NF4 code ("How NF4 works"),
//   Step 4  two 4-bit codes share one byte; the scales are stored beside them.
//
// Layout: B/16 lanes own one block of B elements (B = 32, 64, 128 or 256; 64
// is the pages' example and the default), 16 consecutive elements each (two
// 16-byte loads for bf16, four for fp32); a warp covers 32/(B/16) consecutive
// blocks per iteration and iterates uniformly (the lookup is a warp shuffle).
// The block absmax is a shuffle reduction over the block's lanes.
//
// Nearest code of x = RN(w / a): the number of thresholds (exact code
// midpoints rounded down to fp32) below x.  A 32-bucket table covers [-1, 1];
// lane j of every warp holds bucket j: the one threshold inside it (2.0 if
// none) with the count of thresholds below the bucket in its low 4 mantissa
// bits.  x is first estimated as q = w * RN(1/a) (within 3 * 2^-24 of x); one
// fused multiply-add rounded down puts q's bucket in the low 5 mantissa bits
// of its result, a shuffle fetches the entry, and code = base + (q > entry).
// Elements are decided in pairs with paired fp32 arithmetic (f32x2).
// When q lies within 2^-19 of the entry -- where the estimate, or the 4 bits
// stored in the entry, could change the decision -- the exact quotient
// __fdiv_rn(w, a) is compared with the exact threshold instead.  Every code is
// therefore the one of the IEEE quotient.
#include "nf4_common.cuh"
#include "internal.h"

namespace nf4 {
namespace {

__constant__ uint32_t c_q32[32] = NF4_Q32_INIT;
__constant__ float c_threshold[15] = NF4_THRESHOLD_INIT;
// FP4 (E2M1 / 6): 16 buckets over [0, 1] of |x| and the 7 magnitude thresholds
__constant__ uint32_t c_q16[16] = FP4_Q16_INIT;
__constant__ float c_f4threshold[7] = FP4_THRESHOLD_INIT;

constexpr float kNearThreshold = 0x1p-19f;
constexpr float kTinyScale = 0x1p-120f;  // below this 1/a may overflow: divide exactly

// Exact decision for the rare elements near a threshold (and for blocks whose
// scale is too small for the reciprocal): the IEEE quotient counted against
// the exact thresholds.
__device__ __noinline__ int code_exact(float w, float a) {
  const float x = __fdiv_rn(w, a);
  int code = 0;
#pragma unroll
  for (int i = 0; i < 15; ++i) code += (x > c_threshold[i]) ? 1 : 0;
  return code;
}

// FP4: the magnitude code of |x| against the exact magnitude thresholds, with the sign of x in bit 3 (a zero
// result keeps the sign: -0 is pattern 8)
__device__ __noinline__ int code_exact_fp4(float w, float a) {
  const float x = __fdiv_rn(w, a);
  const float ax = fabsf(x);
  int code = 0;
#pragma unroll
  for (int i = 0; i < 7; ++i) code += (ax > c_f4threshold[i]) ? 1 : 0;
  return code | ((__float_as_uint(x) >> 31) << 3);
}

// FP4 fast path: 16 magnitude buckets (lanes 0..15 of the warp hold them; lanes 16..31 repeat them); q estimates
// w / a within 3 * 2^-24 and has the sign of w
__device__ __forceinline__ uint32_t code_fast_fp4(uint32_t entry, float q, float& gap) {
  const float aq = fabsf(q);
  const float v = __fmaf_rd(aq, 16.0f * NF4_Q32_SCALE, 0x1p23f);  // low 4 mantissa bits: the bucket
  const uint32_t e = __shfl_sync(0xffffffffu, entry, __float_as_int(v));
  const float thr = __uint_as_float(e);
  gap = fminf(gap, fabsf(aq - thr));
  return (e & 15u) + (aq > thr ? 1u : 0u) + ((__float_as_uint(q) >> 31) << 3);
}

// Two elements of NF4 at once: q = w * r and the bucket value v = RD(16 S q + 2^23 + 16) as paired fp32
// operations (each half rounded as its scalar form), two shuffles fetch the bucket entries, and d = thr - q (also
// paired, exact in sign: the difference of two fp32 values is never rounded to zero) gives both the decision
// (q > thr iff d's sign bit is set) and the distance to the threshold.
__device__ __forceinline__ void code_fast_pair(uint32_t entry, float w0, float w1, float r, float& gap,
                                               uint32_t& c0, uint32_t& c1) {
  unsigned long long wq, rr, q, v, d, t;
  asm("mov.b64 %0, {%1, %2};" : "=l"(wq) : "f"(w0), "f"(w1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(rr) : "f"(r));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(q) : "l"(wq), "l"(rr));
  {
    unsigned long long sc, of;
    asm("mov.b64 %0, {%1, %1};" : "=l"(sc) : "f"(16.0f * NF4_Q32_SCALE));
    asm("mov.b64 %0, {%1, %1};" : "=l"(of) : "f"(0x1p23f + 16.0f));
    asm("fma.rm.f32x2 %0, %1, %2, %3;" : "=l"(v) : "l"(q), "l"(sc), "l"(of));
  }
  uint32_t v0, v1;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(v0), "=r"(v1) : "l"(v));
  const uint32_t e0 = __shfl_sync(0xffffffffu, entry, (int)v0);
  const uint32_t e1 = __shfl_sync(0xffffffffu, entry, (int)v1);
  asm("mov.b64 %0, {%1, %2};" : "=l"(t) : "r"(e0), "r"(e1));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(t), "l"(q));
  uint32_t d0, d1;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(d0), "=r"(d1) : "l"(d));
  gap = fminf(gap, fminf(fabsf(__uint_as_float(d0)), fabsf(__uint_as_float(d1))));
  c0 = (e0 & 15u) + (d0 >> 31);
  c1 = (e1 & 15u) + (d1 >> 31);
}

// two codes -> one byte (first in the high nibble); four bytes -> one word
__device__ __forceinline__ uint32_t pack8(const uint32_t (&c)[16], int o) {
  const uint32_t b0 = c[o] * 16u + c[o + 1], b1 = c[o + 2] * 16u + c[o + 3];
  const uint32_t b2 = c[o + 4] * 16u + c[o + 5], b3 = c[o + 6] * 16u + c[o + 7];
  return prmt(prmt(b0, b1, 0x0040), prmt(b2, b3, 0x0040), 0x5410);
}

template <bool kBF16>
__device__ __forceinline__ float load1(const void* src, int64_t i) {
  if (kBF16) return __uint_as_float((uint32_t)(static_cast<const uint16_t*>(src)[i]) << 16);
  return static_cast<const float*>(src)[i];
}

// One warp iteration over the 32 / kL blocks from block wb of one tensor: lane (block wb + lane / kL, part
// lane % kL) loads its 16 consecutive elements (fetch, one iteration ahead) and codes them (code_slice).
template <bool kBF16>
using Raw = uint4[kBF16 ? 2 : 4];

template <bool kBF16, int kL>
__device__ __forceinline__ void fetch(const void* __restrict__ src, int64_t nfull, int64_t wb, int lane,
                                      Raw<kBF16>& raw) {
  constexpr int kB = 16 * kL;
  const int64_t b = wb + lane / kL;
  if (b < nfull) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(src) +
                                                    (b * kB + (lane & (kL - 1)) * 16) * (kBF16 ? 2 : 4));
#pragma unroll
    for (int i = 0; i < (kBF16 ? 2 : 4); ++i) raw[i] = __ldcs(p + i);
  }
}

template <bool kBF16, bool kFp4, int kL>
__device__ __forceinline__ void code_slice(uint32_t entry, int lane, int64_t wb, const void* __restrict__ src,
                                           int64_t n, int64_t nfull, int64_t nblocks, uint8_t* __restrict__ packed,
                                           float* __restrict__ absmax, const Raw<kBF16>& cur) {
  constexpr int kB = 16 * kL;
  const int sub = lane & (kL - 1);  // which 16 of the block
  const int64_t b = wb + lane / kL;
  const bool live = b < nblocks;
  const int64_t first = b * kB + sub * 16;
  float w[16];
  if (live && b < nfull) {
    if (kBF16) {
      const uint32_t u[8] = {cur[0].x, cur[0].y, cur[0].z, cur[0].w, cur[1].x, cur[1].y, cur[1].z, cur[1].w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        w[2 * i] = bf16_lo_to_f32(u[i]);
        w[2 * i + 1] = bf16_hi_to_f32(u[i]);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 v = cur[(kBF16 ? 0 : i)];
        w[4 * i] = __uint_as_float(v.x);
        w[4 * i + 1] = __uint_as_float(v.y);
        w[4 * i + 2] = __uint_as_float(v.z);
        w[4 * i + 3] = __uint_as_float(v.w);
      }
    }
  } else {  // short last block (or no block): missing elements read as 0
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = (live && first + i < n) ? load1<kBF16>(src, first + i) : 0.0f;
  }
  // Step 2: block absmax (exact; max is order-free)
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(w[i]));
#pragma unroll
  for (int off = 1; off < kL; off <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));

  // Step 3: nearest code of RN(w / a); an all-zero block takes the zero code (7)
  const bool zero = !(a > 0.0f);
  const bool exact = !zero && a < kTinyScale;      // 1/a could overflow: divide exactly
  const float r = __frcp_rn(zero ? 1.0f : a);
  uint32_t c[16];
  float gap = 1.0f;
  if (kFp4) {
#pragma unroll
    for (int i = 0; i < 16; ++i) c[i] = code_fast_fp4(entry, __fmul_rn(w[i], r), gap);
  } else {
#pragma unroll
    for (int i = 0; i < 16; i += 2) code_fast_pair(entry, w[i], w[i + 1], r, gap, c[i], c[i + 1]);
  }
  if (exact || gap <= kNearThreshold) {  // rare: redo this lane's 16 elements with exact quotients
#pragma unroll
    for (int i = 0; i < 16; ++i) c[i] = (uint32_t)(kFp4 ? code_exact_fp4(w[i], a) : code_exact(w[i], a));
  }
  // Step 4: element 2j -> high nibble of byte j; an all-zero block is all zero codes (NF4 7, FP4 +0)
  uint32_t lo = pack8(c, 0), hi = pack8(c, 8);
  if (zero) lo = hi = kFp4 ? 0u : 0x77777777u;
  if (!live) return;
  if (b < nfull) {
    *reinterpret_cast<uint2*>(packed + first / 2) = make_uint2(lo, hi);
  } else {
    // short block: write only bytes holding real elements; an odd tail keeps
    // the zero code (NF4 7, FP4 +0) in its low nibble
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t e = first + 2 * j;  // element in the high nibble
      if (e < n) {
        uint8_t v = (uint8_t)((j < 4 ? lo : hi) >> (8 * (j & 3)));
        if (e + 1 >= n) v = (uint8_t)((v & 0xf0u) | (kFp4 ? 0x0u : 0x7u));
        packed[first / 2 + j] = v;
      }
    }
  }
  if (sub == 0) absmax[b] = a;
}

template <bool kBF16, bool kFp4, int kL>
__global__ void __launch_bounds__(256) quantize_kernel(const void* __restrict__ src, int64_t n,
                                                       uint8_t* __restrict__ packed,
                                                       float* __restrict__ absmax) {
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const uint32_t entry = kFp4 ? c_q16[lane & 15] : c_q32[lane];
  // kL lanes own one block of kB = 16 kL elements, 16 consecutive elements each
  constexpr int kB = 16 * kL;
  constexpr int kPerWarp = 32 / kL;                          // blocks per warp and iteration
  const int64_t nfull = n / kB;
  const int64_t nblocks = (n + kB - 1) / kB;
  const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t warp_id = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);

  // raw 16-element slices, one iteration ahead: the next slice's loads are in
  // flight while this one is coded
  Raw<kBF16> cur, nxt;
  int64_t wb = warp_id * kPerWarp;
  pdl_wait();
  if (wb < nblocks) fetch<kBF16, kL>(src, nfull, wb, lane, cur);
  for (; wb < nblocks; wb += warps_total * kPerWarp) {  // uniform per warp
    if (wb + warps_total * kPerWarp < nblocks) fetch<kBF16, kL>(src, nfull, wb + warps_total * kPerWarp, lane, nxt);
    code_slice<kBF16, kFp4, kL>(entry, lane, wb, src, n, nfull, nblocks, packed, absmax, cur);
#pragma unroll
    for (int i = 0; i < (kBF16 ? 2 : 4); ++i) cur[i] = nxt[i];
  }
}

// Several tensors of one dtype and block size: their blocks, each tensor's rounded up to whole warp iterations,
// form one sequence that the warps walk as above (a warp's tensor index only moves forward).
template <bool kBF16, bool kFp4, int kL>
__global__ void __launch_bounds__(256) quantize_many_kernel(const __grid_constant__ QuantManyParams p) {
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const uint32_t entry = kFp4 ? c_q16[lane & 15] : c_q32[lane];
  constexpr int kB = 16 * kL;
  constexpr int kPerWarp = 32 / kL;
  const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
  int64_t W = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);  // warp iteration in the sequence
  pdl_wait();
  if (W >= p.iters) return;
  int t = 0;
  while (t + 1 < p.count && p.item[t + 1].w0 <= W) ++t;
  Raw<kBF16> cur, nxt;
  fetch<kBF16, kL>(p.item[t].src, p.item[t].n / kB, (W - p.item[t].w0) * kPerWarp, lane, cur);
  while (W < p.iters) {
    const QuantItem& it = p.item[t];
    const int64_t wb = (W - it.w0) * kPerWarp;
    W += warps_total;
    if (W < p.iters) {
      int tn = t;
      while (tn + 1 < p.count && p.item[tn + 1].w0 <= W) ++tn;
      fetch<kBF16, kL>(p.item[tn].src, p.item[tn].n / kB, (W - p.item[tn].w0) * kPerWarp, lane, nxt);
      code_slice<kBF16, kFp4, kL>(entry, lane, wb, it.src, it.n, it.n / kB, (it.n + kB - 1) / kB, it.packed,
                                  it.absmax, cur);
      t = tn;
    } else {
      code_slice<kBF16, kFp4, kL>(entry, lane, wb, it.src, it.n, it.n / kB, (it.n + kB - 1) / kB, it.packed,
                                  it.absmax, cur);
    }
#pragma unroll
    for (int i = 0; i < (kBF16 ? 2 : 4); ++i) cur[i] = nxt[i];
  }
}

template <bool kBF16, bool kFp4, int kL>
cudaError_t launch_one(const void* src, int64_t n, uint8_t* packed, float* absmax, cudaStream_t stream, int num_sms) {
  const int64_t nblocks = (n + 16 * kL - 1) / (16 * kL);
  const int per_cta = 256 / kL;
  int64_t grid = (nblocks + per_cta - 1) / per_cta;
  int occ = 0;  // one wave: as many CTAs as fit on the SMs at once
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, quantize_kernel<kBF16, kFp4, kL>, 256, 0) != cudaSuccess ||
      occ < 1)
    occ = 1;
  const int64_t cap = (int64_t)num_sms * occ;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  const cudaError_t e =
      launch_pdl(quantize_kernel<kBF16, kFp4, kL>, dim3((unsigned)grid), dim3(256), 0, stream, src, n, packed, absmax);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <bool kBF16, bool kFp4>
cudaError_t launch_blocks(const void* src, int64_t n, int blocksize, uint8_t* packed, float* absmax,
                          cudaStream_t stream, int num_sms) {
  switch (blocksize) {
    case 32: return launch_one<kBF16, kFp4, 2>(src, n, packed, absmax, stream, num_sms);
    case 64: return launch_one<kBF16, kFp4, 4>(src, n, packed, absmax, stream, num_sms);
    case 128: return launch_one<kBF16, kFp4, 8>(src, n, packed, absmax, stream, num_sms);
    case 256: return launch_one<kBF16, kFp4, 16>(src, n, packed, absmax, stream, num_sms);
    default: return cudaErrorInvalidValue;
  }
}

template <bool kBF16, bool kFp4, int kL>
cudaError_t launch_many_one(QuantManyParams& p, cudaStream_t stream, int num_sms) {
  constexpr int kPerWarp = 32 / kL;
  int64_t iters = 0;
  for (int i = 0; i < p.count; ++i) {
    p.item[i].w0 = iters;
    iters += (p.item[i].n + 16 * kL * kPerWarp - 1) / (16 * kL * kPerWarp);
  }
  p.iters = iters;
  int64_t grid = (iters + 7) / 8;  // 8 warps per CTA
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, quantize_many_kernel<kBF16, kFp4, kL>, 256, 0) !=
          cudaSuccess || occ < 1)
    occ = 1;
  const int64_t cap = (int64_t)num_sms * occ;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  const cudaError_t e = launch_pdl(quantize_many_kernel<kBF16, kFp4, kL>, dim3((unsigned)grid), dim3(256), 0, stream, p);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <bool kBF16, bool kFp4>
cudaError_t launch_many_blocks(QuantManyParams& p, int blocksize, cudaStream_t stream, int num_sms) {
  switch (blocksize) {
    case 32: return launch_many_one<kBF16, kFp4, 2>(p, stream, num_sms);
    case 64: return launch_many_one<kBF16, kFp4, 4>(p, stream, num_sms);
    case 128: return launch_many_one<kBF16, kFp4, 8>(p, stream, num_sms);
    case 256: return launch_many_one<kBF16, kFp4, 16>(p, stream, num_sms);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_quantize_many(QuantManyParams& p, bool bf16, int blocksize, int book, cudaStream_t stream,
                                 int num_sms) {
  if (bf16)
    return book ? launch_many_blocks<true, true>(p, blocksize, stream, num_sms)
                : launch_many_blocks<true, false>(p, blocksize, stream, num_sms);
  return book ? launch_many_blocks<false, true>(p, blocksize, stream, num_sms)
              : launch_many_blocks<false, false>(p, blocksize, stream, num_sms);
}

cudaError_t launch_quantize(const void* src, bool bf16, int64_t n, int blocksize, uint8_t* packed, float* absmax,
                            int book, cudaStream_t stream, int num_sms) {
  if (bf16)
    return book ? launch_blocks<true, true>(src, n, blocksize, packed, absmax, stream, num_sms)
                : launch_blocks<true, false>(src, n, blocksize, packed, absmax, stream, num_sms);
  return book ? launch_blocks<false, true>(src, n, blocksize, packed, absmax, stream, num_sms)
              : launch_blocks<false, false>(src, n, blocksize, packed, absmax, stream, num_sms);
}

}  // namespace nf4
