// quantize.cu -- blockwise NF4 quantization (level 1).
//
// "bitsandbytes" (ozercemkelahmet.com/tools), "How it works":
//   Step 1  blocks of 64 consecutive values,
//   Step 2  the block's absmax is its scale; every value is divided by it,
//   Step 3  each scaled value takes the nearest NF4 code ("How NF4 works"),
//   Step 4  two 4-bit codes share one byte; the scales are stored beside them.
//
// Layout: four lanes own one 64-element block, 16 consecutive elements each
// (two 16-byte loads for bf16, four for fp32).  The block absmax is a 4-lane
// shuffle reduction.  The nearest code of x = RN(w / a) is the number of
// thresholds below x; a 514-entry bucket table in shared memory turns that
// into one lookup and one compare.  x is first estimated as w * RN(1/a); when
// the estimate lies within 2^-19 of the bucket's threshold (where the estimate
// and the IEEE quotient could fall on different sides) the exact quotient
// __fdiv_rn(w, a) decides, so every code equals the one of the IEEE quotient.
#include "nf4_common.cuh"
#include "internal.h"

namespace nf4 {
namespace {

__constant__ float c_bucket_thr[NF4_NUM_BUCKETS] = NF4_BUCKET_THRESHOLD_INIT;
__constant__ unsigned char c_bucket_base[NF4_NUM_BUCKETS] = NF4_BUCKET_BASE_INIT;

struct Bucket {
  float thr;
  int base;
};

constexpr float kNearThreshold = 0x1p-19f;   // estimate is within 3 * 2^-24 of the quotient
constexpr float kTinyScale = 0x1p-120f;      // below this 1/a may overflow: divide exactly

__device__ __forceinline__ int code_of(const Bucket* tab, float w, float a, float r, bool exact) {
  float q = exact ? __fdiv_rn(w, a) : __fmul_rn(w, r);
  float v = __fmaf_rn(q, 0.5f, NF4_BUCKET_BIAS);
  unsigned bk = (unsigned)((__float_as_int(v) >> NF4_BUCKET_SHIFT) - (0x40000000 >> NF4_BUCKET_SHIFT));
  bk = min(bk, (unsigned)(NF4_NUM_BUCKETS - 1));  // NaN/Inf inputs stay in bounds
  Bucket e = tab[bk];
  int code = e.base + (q > e.thr ? 1 : 0);
  if (!exact && fabsf(q - e.thr) <= kNearThreshold) {
    float x = __fdiv_rn(w, a);
    code = e.base + (x > e.thr ? 1 : 0);
  }
  return code;
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
  __shared__ Bucket tab[NF4_NUM_BUCKETS];
  for (int i = threadIdx.x; i < NF4_NUM_BUCKETS; i += blockDim.x) tab[i] = Bucket{c_bucket_thr[i], (int)c_bucket_base[i]};
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int sub = lane & 3;                                  // which 16 of the block's 64
  const unsigned gmask = 0xfu << (lane & ~3);                // the 4 lanes of this block
  const int64_t nfull = n / kBlock;
  const int64_t nblocks = (n + kBlock - 1) / kBlock;
  const int64_t stride = (int64_t)gridDim.x * (blockDim.x / 4);

  for (int64_t b = (int64_t)blockIdx.x * (blockDim.x / 4) + (threadIdx.x >> 2); b < nblocks; b += stride) {
    const int64_t first = b * kBlock + sub * 16;
    float w[16];
    if (b < nfull) {
      load16<kBF16>(src, first, w);
    } else {  // short last block: missing elements read as 0 (they do not change the absmax)
#pragma unroll
      for (int i = 0; i < 16; ++i) w[i] = (first + i < n) ? load1<kBF16>(src, first + i) : 0.0f;
    }
    // Step 2: block absmax (exact; max is order-free)
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(w[i]));
    a = fmaxf(a, __shfl_xor_sync(gmask, a, 1));
    a = fmaxf(a, __shfl_xor_sync(gmask, a, 2));

    // Step 3: nearest code of RN(w / a); all-zero block -> zero code (7)
    uint32_t lo = 0x77777777u, hi = 0x77777777u;
    if (a > 0.0f) {
      const bool exact = a < kTinyScale;
      const float r = exact ? 0.0f : __frcp_rn(a);
      int c[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) c[i] = code_of(tab, w[i], a, r, exact);
      // Step 4: element 2j -> high nibble of byte j
      lo = 0;
      hi = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        lo |= (uint32_t)((c[2 * j] << 4) | c[2 * j + 1]) << (8 * j);
        hi |= (uint32_t)((c[8 + 2 * j] << 4) | c[8 + 2 * j + 1]) << (8 * j);
      }
    }
    if (b < nfull) {
      *reinterpret_cast<uint2*>(packed + first / 2) = make_uint2(lo, hi);
    } else {
      // short block: write only the bytes that hold real elements; an odd
      // tail keeps the zero code (7) in its low nibble
      const int64_t nbytes = (n + 1) / 2;
      uint8_t bytes[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        bytes[j] = (uint8_t)(lo >> (8 * j));
        bytes[4 + j] = (uint8_t)(hi >> (8 * j));
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t e = first + 2 * j;  // element in the high nibble
        if (e < n) {
          uint8_t v = bytes[j];
          if (e + 1 >= n) v = (uint8_t)((v & 0xf0u) | 0x7u);
          if (first / 2 + j < nbytes) packed[first / 2 + j] = v;
        }
      }
    }
    if (sub == 0) absmax[b] = a;
  }
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
  return cudaGetLastError();
}

}  // namespace nf4
