// double_quant.cu -- double quantization of the level-1 absmax array.
//
// "bitsandbytes quantization tutorial" (mljourney.com), "How NF4 Works": the
// per-block scale constants are themselves quantized from float32 to float8;
// "bitsandbytes" (ozercemkelahmet.com/tools), "Double quantization".  The
// second level reuses the level-1 recipe with an 8-bit code book, in the order
// of that page's "A worked example": block absmax m, x = RN(r / m),
// y = RN(x * Q), code = round(y) -- E4M3 (Q = 448, nearest-even, saturating)
// or int8 (Q = 127, half away from zero, clamped).  The mean is removed first
// (one fp32 per tensor): mu = fp32(fp64(exact sum) / nb).
//
// Two kernels, chained with programmatic dependent launch (no grid barrier):
//   sum     every fp32 value is an integer multiple of 2^-149, so each thread
//           adds its values into ten signed 64-bit limbs holding 32 bits each
//           of a 320-bit fixed-point number; integer addition makes the total
//           exact and independent of order.  Warp shuffles and shared memory
//           combine threads, 64-bit atomics combine CTAs.  The CTA that
//           arrives last (a counter in the workspace) normalises the limbs,
//           rounds the sum once to fp64, writes mu and resets the limbs and
//           the counter, so the workspace is ready for the next call (only the
//           first call needs a zeroed buffer).
//   encode  one warp per 256-value block: residuals, block absmax, codes; it
//           reads mu after waiting for the sum kernel.
#include "nf4_common.cuh"
#include "internal.h"

namespace nf4 {
namespace {

constexpr int kLimbs = 10;

struct SumWorkspace {
  unsigned long long limb[kLimbs];  // two's-complement running sums of 32-bit digits
  unsigned int count;               // CTAs of the running sum that have added their share
};
static_assert(sizeof(SumWorkspace) <= kDoubleQuantWorkspace, "workspace");

__device__ __forceinline__ void add_value(long long (&acc)[kLimbs], float x) {
  const uint32_t u = __float_as_uint(x);
  const uint32_t e = (u >> 23) & 0xffu, f = u & 0x7fffffu;
  const uint32_t mant = e ? (f | 0x800000u) : f;  // value = mant * 2^(sh - 149)
  const int sh = e ? (int)e - 1 : 0;
  const int li = sh >> 5;
  const uint64_t v = (uint64_t)mant << (sh & 31);
  long long lo = (long long)(v & 0xffffffffull), hi = (long long)(v >> 32);
  if (u >> 31) {
    lo = -lo;
    hi = -hi;
  }
#pragma unroll
  for (int L = 0; L < kLimbs; ++L) acc[L] += (L == li) ? lo : ((L == li + 1) ? hi : 0);
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

// Exact sum of the absmax values; the last CTA derives mu, writes it and resets the workspace.
__global__ void __launch_bounds__(256) dq_sum_kernel(const float* __restrict__ a, int64_t nb,
                                                     float* __restrict__ mean_out, SumWorkspace* __restrict__ ws) {
  pdl_launch_dependents();  // the encode kernel may set itself up; it waits for this one to finish
  pdl_wait();
  long long acc[kLimbs];
#pragma unroll
  for (int L = 0; L < kLimbs; ++L) acc[L] = 0;
  const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t n4 = nb / 4;  // absmax is 16-byte aligned: float4 loads for the body
  for (int64_t i = tid; i < n4; i += nthreads) {
    const float4 v = reinterpret_cast<const float4*>(a)[i];
    add_value(acc, v.x);
    add_value(acc, v.y);
    add_value(acc, v.z);
    add_value(acc, v.w);
  }
  for (int64_t i = 4 * n4 + tid; i < nb; i += nthreads) add_value(acc, a[i]);
#pragma unroll
  for (int L = 0; L < kLimbs; ++L)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[L] += __shfl_xor_sync(0xffffffffu, acc[L], off);
  __shared__ long long red[8][kLimbs];
  __shared__ int s_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0)
#pragma unroll
    for (int L = 0; L < kLimbs; ++L) red[warp][L] = acc[L];
  __syncthreads();
  if (threadIdx.x < kLimbs) {
    long long t = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w][threadIdx.x];
    // values of similar magnitude touch two or three limbs: skip the zero ones (all limbs share one cache line)
    if (t != 0) atomicAdd(&ws->limb[threadIdx.x], (unsigned long long)t);  // wraps mod 2^64 = signed add
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&ws->count, 1u) == gridDim.x - 1;
  __syncthreads();
  if (s_last && threadIdx.x == 0) {  // every other CTA has added its share
    __threadfence();
    long long l[kLimbs];
#pragma unroll
    for (int L = 0; L < kLimbs; ++L) l[L] = (long long)atomicExch(&ws->limb[L], 0ull);  // read and reset
    *mean_out = finish_mean(l, nb);
    ws->count = 0;
  }
}

// Codes: one warp per block of kDqBlock residuals.
__global__ void __launch_bounds__(256) dq_encode_kernel(const float* __restrict__ a, int64_t nb, int dq_code,
                                                        uint8_t* __restrict__ q, float* __restrict__ scale,
                                                        const float* __restrict__ mean) {
  pdl_launch_dependents();
  pdl_wait();  // the sum kernel has finished: mu is in memory
  const float mu = *mean;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ngroups = (nb + kDqBlock - 1) / kDqBlock;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const float Q = dq_code == 0 ? kE4M3Top : kInt8Top;
  for (int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp; g < ngroups; g += nwarps) {
    const int64_t first = g * kDqBlock + lane * 8;
    const bool full = (g + 1) * kDqBlock <= nb;
    float r[8];
    if (full) {
      const float4* p = reinterpret_cast<const float4*>(a + first);
      const float4 v0 = p[0], v1 = p[1];
      r[0] = v0.x; r[1] = v0.y; r[2] = v0.z; r[3] = v0.w;
      r[4] = v1.x; r[5] = v1.y; r[6] = v1.z; r[7] = v1.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) r[i] = (first + i < nb) ? a[first + i] : mu;  // mu -> residual 0
    }
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      r[i] = __fsub_rn(r[i], mu);  // residual after removing the mean
      m = fmaxf(m, fabsf(r[i]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) scale[g] = m;
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = (m != 0.0f) ? __fmul_rn(__fdiv_rn(r[i], m), Q) : 0.0f;
    uint32_t lo, hi;
    if (dq_code == 0) {
      lo = pack_e4m3x2(y[0], y[1]) | (pack_e4m3x2(y[2], y[3]) << 16);
      hi = pack_e4m3x2(y[4], y[5]) | (pack_e4m3x2(y[6], y[7]) << 16);
    } else {
      uint32_t bb[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float t = fminf(fmaxf(roundf(y[i]), -127.0f), 127.0f);  // half away from zero, clamp
        bb[i] = (uint32_t)(uint8_t)(int8_t)(int)t;
      }
      lo = bb[0] | (bb[1] << 8) | (bb[2] << 16) | (bb[3] << 24);
      hi = bb[4] | (bb[5] << 8) | (bb[6] << 16) | (bb[7] << 24);
    }
    if (full) {
      *reinterpret_cast<uint2*>(q + first) = make_uint2(lo, hi);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (first + i < nb) q[first + i] = (uint8_t)((i < 4 ? lo : hi) >> (8 * (i & 3)));
    }
  }
}

}  // namespace

cudaError_t launch_double_quant(const float* absmax, int64_t nb, int dq_code, uint8_t* q, float* scale,
                                float* mean, void* workspace, bool clear, unsigned* /*err*/, cudaStream_t stream,
                                int num_sms) {
  cudaError_t e = cudaSuccess;
  if (clear && (e = cudaMemsetAsync(workspace, 0, sizeof(SumWorkspace), stream)) != cudaSuccess) return e;
  auto* ws = static_cast<SumWorkspace*>(workspace);
  // sum: each thread at least 16 values (fewer CTAs, fewer atomics on the limbs), at most one CTA per SM
  int64_t grid = (nb + 256 * 16 - 1) / (256 * 16);
  grid = grid < 1 ? 1 : (grid > num_sms ? num_sms : grid);
  e = launch_pdl(dq_sum_kernel, dim3((unsigned)grid), dim3(256), 0, stream, absmax, nb, mean, ws);
  count_launches(1);
  if (e != cudaSuccess) return e;
  // encode: one warp per 256-value block, up to 8 CTAs of 8 warps per SM
  const int64_t ngroups = (nb + kDqBlock - 1) / kDqBlock;
  int64_t grid2 = (ngroups + 7) / 8;
  grid2 = grid2 < 1 ? 1 : (grid2 > 8 * (int64_t)num_sms ? 8 * (int64_t)num_sms : grid2);
  e = launch_pdl(dq_encode_kernel, dim3((unsigned)grid2), dim3(256), 0, stream, (const float*)absmax, nb, dq_code, q,
                 scale, (const float*)mean);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace nf4

