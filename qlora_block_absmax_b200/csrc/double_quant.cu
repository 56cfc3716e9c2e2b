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
#include "exact_sum.cuh"
#include "internal.h"

namespace nf4 {
namespace {

static_assert(sizeof(SumWorkspace) <= kDoubleQuantWorkspace, "workspace");

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
  e = launch_pdl(dq_encode_kernel, dim3((unsigned)grid2), dim3(256), 0, stream, (const float*)absmax, nb,
                 dq_code, q, scale, (const float*)mean);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace nf4

