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
// Two kernels, chained with programmatic dependent launch (no grid barrier),
// for one array or (the "many" pair) for up to 256 arrays at once, each with
// its own mean:
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
#include "exact_sum.cuh"
#include "internal.h"

namespace nf4 {
namespace {

static_assert(sizeof(SumWorkspace) <= kDoubleQuantWorkspace, "workspace");

// Add the float4 run a4[0, n4) to this thread's runner, thread `tid` of `nthreads` taking every nthreads-th
// vector: four loads in flight per thread before their sixteen values are added.
__device__ __forceinline__ void sum_body(Runner& r, const float4* __restrict__ a4, int64_t n4, int64_t tid,
                                         int64_t nthreads, long long* limbs) {
  int64_t i = tid;
  for (; i + 3 * nthreads < n4; i += 4 * nthreads) {
    const float4 v0 = __ldcs(a4 + i), v1 = __ldcs(a4 + i + nthreads), v2 = __ldcs(a4 + i + 2 * nthreads),
                 v3 = __ldcs(a4 + i + 3 * nthreads);
    const float v[16] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w, v2.x, v2.y, v2.z, v2.w, v3.x, v3.y, v3.z, v3.w};
#pragma unroll
    for (int k = 0; k < 16; ++k) runner_add(r, v[k], limbs);
  }
  for (; i < n4; i += nthreads) {
    const float4 v = __ldcs(a4 + i);
    runner_add(r, v.x, limbs);
    runner_add(r, v.y, limbs);
    runner_add(r, v.z, limbs);
    runner_add(r, v.w, limbs);
  }
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
  sum_body(r, reinterpret_cast<const float4*>(a), n4, tid, nthreads, limbs);
  for (int64_t i = 4 * n4 + tid; i < nb; i += nthreads) runner_add(r, a[i], limbs);
  runner_warp_flush(r, limbs);
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

// ------------------------------------------------------------------ several tensors per launch

// Per tensor: the running limbs and how many of its values the CTAs have added (the CTA whose share completes
// the count derives mu and resets the record).
struct ManyRecord {
  unsigned long long limb[kLimbs];
  unsigned long long done;
};
static_assert(sizeof(ManyRecord) <= kDqManyRecord, "workspace record");

// the item holding element x (by = 0) or 256-block x (by = 1) of the concatenation: the last with start <= x
__device__ __forceinline__ int find_item(const DqManyParams& p, int64_t x, int by) {
  int lo = 0, hi = p.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    const int64_t start = by ? p.item[mid].g0 : p.item[mid].e0;
    if (start <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The sum kernel over the concatenation of all arrays: CTA c takes the equal share [c T / G, (c + 1) T / G) of the
// T values and sums its part of each array it meets separately (the same exact digits as the one-array kernel).
__global__ void __launch_bounds__(512) dq_sum_many_kernel(const __grid_constant__ DqManyParams p,
                                                          ManyRecord* __restrict__ ws) {
  __shared__ long long limbs[kLimbs];
  if (threadIdx.x < kLimbs) limbs[threadIdx.x] = 0;
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();  // (after the wait, as in the one-array kernel: the encode grid may read the arrays early)
  const int64_t lo = p.total * blockIdx.x / gridDim.x, hi = p.total * (blockIdx.x + 1) / gridDim.x;
  if (lo >= hi) return;
  for (int t = find_item(p, lo, 0); t < p.count && p.item[t].e0 < hi; ++t) {
    const float* __restrict__ a = p.item[t].a;
    const int64_t nb = p.item[t].nb, e0 = p.item[t].e0;
    const int64_t l0 = (lo > e0 ? lo : e0) - e0;
    const int64_t l1 = (hi < e0 + nb ? hi : e0 + nb) - e0;
    Runner r;
    const int64_t b0 = ((l0 + 3) & ~(int64_t)3) < l1 ? ((l0 + 3) & ~(int64_t)3) : l1;  // float4 body from here
    const int64_t n4 = (l1 - b0) >> 2;
    for (int64_t i = l0 + threadIdx.x; i < b0; i += blockDim.x) runner_add(r, a[i], limbs);
    sum_body(r, reinterpret_cast<const float4*>(a + b0), n4, threadIdx.x, blockDim.x, limbs);
    for (int64_t i = b0 + 4 * n4 + threadIdx.x; i < l1; i += blockDim.x) runner_add(r, a[i], limbs);
    runner_warp_flush(r, limbs);
    __syncthreads();
    if (threadIdx.x < 32) {
      if (threadIdx.x < kLimbs) {
        const long long v = limbs[threadIdx.x];
        if (v != 0) atomicAdd(&ws[t].limb[threadIdx.x], (unsigned long long)v);
        __threadfence();  // the limb additions before the count below
      }
      __syncwarp();
      if (threadIdx.x == 0) {
        const unsigned long long seg = (unsigned long long)(l1 - l0);
        if (atomicAdd(&ws[t].done, seg) + seg == (unsigned long long)nb) {  // every other share is in
          __threadfence();
          long long l[kLimbs];
#pragma unroll
          for (int L = 0; L < kLimbs; ++L) l[L] = (long long)atomicExch(&ws[t].limb[L], 0ull);  // read and reset
          *p.item[t].mean = finish_mean(l, nb);
          ws[t].done = 0;
        }
      }
    }
    __syncthreads();  // warp 0 has read the shared limbs
    if (threadIdx.x < kLimbs) limbs[threadIdx.x] = 0;
    __syncthreads();
  }
}

// Codes for every 256-block of every array, one warp per block; as the one-array encode kernel, with the block's
// array found by its index and that array's mu read after the wait.
__global__ void __launch_bounds__(256) dq_encode_many_kernel(const __grid_constant__ DqManyParams p, int dq_code) {
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const float Q = dq_code == 0 ? kE4M3Top : kInt8Top;
  int64_t G = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
  if (G >= p.groups) {
    pdl_wait();  // a warp without a block still orders itself after the sum kernel
    return;
  }
  // this warp's blocks G, G + nwarps, ... in increasing order: the array index only moves forward, and the next
  // block's values are loaded before the current block is encoded
  int t = find_item(p, G, 1);
  auto load = [&](int64_t g, const DqItem& it, float (&r)[8]) {
    const int64_t first = g * kDqBlock + lane * 8;
    if ((g + 1) * kDqBlock <= it.nb) {
      const float4* ptr = reinterpret_cast<const float4*>(it.a + first);
      const float4 v0 = __ldcg(ptr), v1 = __ldcg(ptr + 1);
      r[0] = v0.x; r[1] = v0.y; r[2] = v0.z; r[3] = v0.w;
      r[4] = v1.x; r[5] = v1.y; r[6] = v1.z; r[7] = v1.w;
    }
  };
  float nxt[8];
  load(G - p.item[t].g0, p.item[t], nxt);
  pdl_wait();  // the sum kernel has finished: every mu is in memory
  while (G < p.groups) {
    const DqItem& it = p.item[t];
    const int64_t g = G - it.g0, nb = it.nb;
    float r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) r[i] = nxt[i];
    // the next block of this warp
    G += nwarps;
    if (G < p.groups) {
      int tn = t;
      while (tn + 1 < p.count && p.item[tn + 1].g0 <= G) ++tn;
      load(G - p.item[tn].g0, p.item[tn], nxt);
      t = tn;
    }
    const int64_t first = g * kDqBlock + lane * 8;
    const bool full = (g + 1) * kDqBlock <= nb;
    const float mu = __ldcg(it.mean);
    if (!full) {
#pragma unroll
      for (int i = 0; i < 8; ++i) r[i] = (first + i < nb) ? __ldcg(it.a + first + i) : mu;  // mu -> residual 0
    }
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      r[i] = __fsub_rn(r[i], mu);
      m = fmaxf(m, fabsf(r[i]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) it.scale[g] = m;
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
        const float tq = fminf(fmaxf(roundf(y[i]), -127.0f), 127.0f);  // half away from zero, clamp
        bb[i] = (uint32_t)(uint8_t)(int8_t)(int)tq;
      }
      lo = bb[0] | (bb[1] << 8) | (bb[2] << 16) | (bb[3] << 24);
      hi = bb[4] | (bb[5] << 8) | (bb[6] << 16) | (bb[7] << 24);
    }
    if (full) {
      *reinterpret_cast<uint2*>(it.q + first) = make_uint2(lo, hi);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (first + i < nb) it.q[first + i] = (uint8_t)((i < 4 ? lo : hi) >> (8 * (i & 3)));
    }
  }
}

}  // namespace

cudaError_t launch_double_quant_many(const DqManyParams& p, int dq_code, void* workspace, cudaStream_t stream,
                                     int num_sms) {
  int64_t grid = (p.total + 512 * 4 - 1) / (512 * 4);  // two CTAs of 512 per SM at most
  grid = grid < 1 ? 1 : (grid > 2 * (int64_t)num_sms ? 2 * (int64_t)num_sms : grid);
  cudaError_t e = launch_pdl(dq_sum_many_kernel, dim3((unsigned)grid), dim3(512), 0, stream, p,
                             static_cast<ManyRecord*>(workspace));
  count_launches(1);
  if (e != cudaSuccess) return e;
  int64_t grid2 = (p.groups + 7) / 8;
  grid2 = grid2 < 1 ? 1 : (grid2 > 8 * (int64_t)num_sms ? 8 * (int64_t)num_sms : grid2);
  e = launch_pdl(dq_encode_many_kernel, dim3((unsigned)grid2), dim3(256), 0, stream, p, dq_code);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

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
  e = launch_pdl(dq_encode_kernel, dim3((unsigned)grid2), dim3(256), 0, stream, (const float*)absmax, nb,
                 dq_code, q, scale, (const float*)mean);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace nf4

