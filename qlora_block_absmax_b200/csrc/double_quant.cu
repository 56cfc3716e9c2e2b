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
//   sum     every fp32 value is an integer multiple of 2^-149: a 56-bit chunk
//           at one of ten 32-bit limbs of a 320-bit fixed-point number.  Each
//           thread adds its chunks into two 64-bit registers (the limb of its
//           first value and the next one; others go straight to shared
//           memory), then hands 32-bit digits on; integer addition makes the
//           total exact and independent of order.  Warp shuffles and shared
//           memory combine threads, 64-bit atomics combine CTAs.  The CTA that
//           arrives last (a counter in the workspace) normalises the limbs,
//           rounds the sum once to fp64, writes mu and resets the limbs and
//           the counter, so the workspace is ready for the next call (only the
//           first call needs a zeroed buffer).
//   encode  one warp per 256-value block: residuals, block absmax, codes.  It
//           loads its absmax values while the sum kernel still runs (that
//           kernel lets it start only once the array is complete) and waits
//           for the sum kernel only before reading mu.
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

// Exact sum of the absmax values; the last CTA derives mu, writes it and resets the workspace.
__global__ void __launch_bounds__(512) dq_sum_kernel(const float* __restrict__ a, int64_t nb,
                                                     float* __restrict__ mean_out, SumWorkspace* __restrict__ ws) {
  __shared__ long long limbs[kLimbs];
  if (threadIdx.x < kLimbs) limbs[threadIdx.x] = 0;
  __syncthreads();
  pdl_wait();
  // Signalled only now that the grid before this one (the producer of `a`) has finished: the encode kernel may
  // then read `a` before its own wait, which only has to cover mu.
  pdl_launch_dependents();
  Runner r;
  const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t n4 = nb / 4;  // absmax is 16-byte aligned: float4 loads for the body
  for (int64_t i = tid; i < n4; i += nthreads) {
    const float4 v = __ldcs(reinterpret_cast<const float4*>(a) + i);
    runner_add(r, v.x, limbs);
    runner_add(r, v.y, limbs);
    runner_add(r, v.z, limbs);
    runner_add(r, v.w, limbs);
  }
  for (int64_t i = 4 * n4 + tid; i < nb; i += nthreads) runner_add(r, a[i], limbs);
  // combine the warp's runners: one set of digits when every lane has the same base (the usual case)
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
  __syncthreads();
  if (threadIdx.x < 32) {  // warp 0 alone hands the CTA's limbs on and counts the CTA in
    if (threadIdx.x < kLimbs) {
      const long long t = limbs[threadIdx.x];
      // values of similar magnitude touch two or three limbs: skip the zero ones (all limbs share one cache line)
      if (t != 0) atomicAdd(&ws->limb[threadIdx.x], (unsigned long long)t);  // wraps mod 2^64 = signed add
      __threadfence();  // the limb additions before the count below
    }
    __syncwarp();
    if (threadIdx.x == 0 && atomicAdd(&ws->count, 1u) == gridDim.x - 1) {  // every other CTA has added its share
      __threadfence();
      long long l[kLimbs];
#pragma unroll
      for (int L = 0; L < kLimbs; ++L) l[L] = (long long)atomicExch(&ws->limb[L], 0ull);  // read and reset
      *mean_out = finish_mean(l, nb);
      ws->count = 0;
    }
  }
}

// Codes: one warp per block of kDqBlock residuals.  The sum kernel signals its dependents only after its own
// wait, so by the time this grid starts the absmax array is complete: its values are loaded (at L2, not through
// a possibly older L1 line) before the wait, which then covers only mu.
__global__ void __launch_bounds__(256) dq_encode_kernel(const float* __restrict__ a, int64_t nb, int dq_code,
                                                        uint8_t* __restrict__ q, float* __restrict__ scale,
                                                        const float* __restrict__ mean) {
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ngroups = (nb + kDqBlock - 1) / kDqBlock;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const float Q = dq_code == 0 ? kE4M3Top : kInt8Top;
  bool waited = false;
  float mu = 0.0f;
  for (int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp; g < ngroups; g += nwarps) {
    const int64_t first = g * kDqBlock + lane * 8;
    const bool full = (g + 1) * kDqBlock <= nb;
    float r[8];
    if (full) {
      const float4* p = reinterpret_cast<const float4*>(a + first);
      const float4 v0 = __ldcg(p), v1 = __ldcg(p + 1);
      r[0] = v0.x; r[1] = v0.y; r[2] = v0.z; r[3] = v0.w;
      r[4] = v1.x; r[5] = v1.y; r[6] = v1.z; r[7] = v1.w;
    }
    if (!waited) {  // the sum kernel has finished: mu is in memory
      pdl_wait();
      mu = __ldcg(mean);
      waited = true;
    }
    if (!full) {
#pragma unroll
      for (int i = 0; i < 8; ++i) r[i] = (first + i < nb) ? __ldcg(a + first + i) : mu;  // mu -> residual 0
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
  if (!waited) pdl_wait();  // a warp without a block still orders itself after the sum kernel
}

}  // namespace

cudaError_t launch_double_quant(const float* absmax, int64_t nb, int dq_code, uint8_t* q, float* scale,
                                float* mean, void* workspace, bool clear, unsigned* /*err*/, cudaStream_t stream,
                                int num_sms) {
  cudaError_t e = cudaSuccess;
  if (clear && (e = cudaMemsetAsync(workspace, 0, sizeof(SumWorkspace), stream)) != cudaSuccess) return e;
  auto* ws = static_cast<SumWorkspace*>(workspace);
  // sum: one CTA of 512 threads per SM at most (one set of global limb atomics per CTA), at least 4 values a thread
  int64_t grid = (nb + 512 * 4 - 1) / (512 * 4);
  grid = grid < 1 ? 1 : (grid > num_sms ? num_sms : grid);
  e = launch_pdl(dq_sum_kernel, dim3((unsigned)grid), dim3(512), 0, stream, absmax, nb, mean, ws);
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

