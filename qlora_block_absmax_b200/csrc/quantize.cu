// quantize.cu -- blockwise NF4 quantization (level 1).
//
// "bitsandbytes" (ozercemkelahmet.com/tools), "How it works":
//   Step 1  blocks of 64 consecutive values,
//   Step 2  the block's absmax is its scale; every value is divided by it,
//   Step 3  each scaled value takes the nearest NF4 code ("How NF4 works"),
//   Step 4  two 4-bit codes share one byte; the scales are stored beside them.
//
// Layout: four lanes own one 64-element block, 16 consecutive elements each
// (two 16-byte loads for bf16, four for fp32); a warp covers 8 consecutive
// blocks per iteration and iterates uniformly (the lookup is a warp shuffle).
// The block absmax is a 4-lane shuffle reduction.
//
// Nearest code of x = RN(w / a): the number of thresholds (exact code
// midpoints rounded down to fp32) below x.  A 32-bucket table covers [-1, 1];
// lane j of every warp holds bucket j: the one threshold inside it (2.0 if
// none) with the count of thresholds below the bucket in its low 4 mantissa
// bits.  x is first estimated as q = w * RN(1/a) (within 3 * 2^-24 of x); q
// picks the bucket, a shuffle fetches the entry, and code = base + (q > entry).
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

// `entry` is this lane's bucket word; every lane of the warp must call this
// (the lookup is a shuffle).  q estimates w / a within 3 * 2^-24.  `near`
// records whether the estimate was too close to the entry to decide.
__device__ __forceinline__ int code_fast(uint32_t entry, float q, bool& near) {
  const float v = __fmaf_rn(q, NF4_Q32_SCALE, 3.0f);
  // lane index wraps modulo 32, so the exponent bits above the bucket need no mask
  const uint32_t e = __shfl_sync(0xffffffffu, entry, __float_as_int(v) >> 18);
  const float thr = __uint_as_float(e);
  near |= fabsf(q - thr) <= kNearThreshold;
  return (int)(e & 15u) + (q > thr ? 1 : 0);
}

template <bool kBF16>
__device__ __forceinline__ void load16(const void* src, int64_t first, float (&w)[16]) {
  if (kBF16) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(src) + first);
    uint4 v0 = __ldcs(p), v1 = __ldcs(p + 1);
    uint32_t u[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w[2 * i] = bf16_lo_to_f32(u[i]);
      w[2 * i + 1] = bf16_hi_to_f32(u[i]);
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(src) + first);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 v = __ldcs(p + i);
      w[4 * i] = v.x;
      w[4 * i + 1] = v.y;
      w[4 * i + 2] = v.z;
      w[4 * i + 3] = v.w;
    }
  }
}

template <bool kBF16>
__device__ __forceinline__ float load1(const void* src, int64_t i) {
  if (kBF16) return __uint_as_float((uint32_t)(static_cast<const uint16_t*>(src)[i]) << 16);
  return static_cast<const float*>(src)[i];
}

template <bool kBF16>
__global__ void __launch_bounds__(256) quantize_kernel(const void* __restrict__ src, int64_t n,
                                                       uint8_t* __restrict__ packed,
                                                       float* __restrict__ absmax) {
  const int lane = threadIdx.x & 31;
  const uint32_t entry = c_q32[lane];
  const int sub = lane & 3;                                  // which 16 of the block's 64
  const unsigned gmask = 0xfu << (lane & ~3);                // the 4 lanes of this block
  const int64_t nfull = n / kBlock;
  const int64_t nblocks = (n + kBlock - 1) / kBlock;
  const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t warp_id = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);

  for (int64_t wb = warp_id * 8; wb < nblocks; wb += warps_total * 8) {  // uniform per warp
    const int64_t b = wb + (lane >> 2);
    const bool live = b < nblocks;
    const int64_t first = b * kBlock + sub * 16;
    float w[16];
    if (live && b < nfull) {
      load16<kBF16>(src, first, w);
    } else {  // short last block (or no block): missing elements read as 0
#pragma unroll
      for (int i = 0; i < 16; ++i) w[i] = (live && first + i < n) ? load1<kBF16>(src, first + i) : 0.0f;
    }
    // Step 2: block absmax (exact; max is order-free)
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(w[i]));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));

    // Step 3: nearest code of RN(w / a); an all-zero block takes the zero code (7)
    const bool zero = !(a > 0.0f);
    const bool exact = !zero && a < kTinyScale;      // 1/a could overflow: divide exactly
    const float r = __frcp_rn(zero ? 1.0f : a);
    int c[16];
    bool near = exact;
#pragma unroll
    for (int i = 0; i < 16; ++i) c[i] = code_fast(entry, __fmul_rn(w[i], r), near);
    if (near) {  // rare: redo this lane's 16 elements with exact quotients
#pragma unroll
      for (int i = 0; i < 16; ++i) c[i] = code_exact(w[i], a);
    }
    // Step 4: element 2j -> high nibble of byte j
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      lo |= (uint32_t)((c[2 * j] << 4) | c[2 * j + 1]) << (8 * j);
      hi |= (uint32_t)((c[8 + 2 * j] << 4) | c[8 + 2 * j + 1]) << (8 * j);
    }
    if (zero) lo = hi = 0x77777777u;
    if (!live) continue;
    if (b < nfull) {
      *reinterpret_cast<uint2*>(packed + first / 2) = make_uint2(lo, hi);
    } else {
      // short block: write only bytes holding real elements; an odd tail keeps
      // the zero code (7) in its low nibble
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t e = first + 2 * j;  // element in the high nibble
        if (e < n) {
          uint8_t v = (uint8_t)((j < 4 ? lo : hi) >> (8 * (j & 3)));
          if (e + 1 >= n) v = (uint8_t)((v & 0xf0u) | 0x7u);
          packed[first / 2 + j] = v;
        }
      }
    }
    if (sub == 0) absmax[b] = a;
  }
  (void)gmask;
}

}  // namespace

cudaError_t launch_quantize(const void* src, bool bf16, int64_t n, uint8_t* packed, float* absmax,
                            cudaStream_t stream, int num_sms) {
  const int64_t nblocks = (n + kBlock - 1) / kBlock;
  const int per_cta = 256 / 4;
  int64_t grid = (nblocks + per_cta - 1) / per_cta;
  const int64_t cap = (int64_t)num_sms * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  if (bf16)
    quantize_kernel<true><<<(unsigned)grid, 256, 0, stream>>>(src, n, packed, absmax);
  else
    quantize_kernel<false><<<(unsigned)grid, 256, 0, stream>>>(src, n, packed, absmax);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace nf4
