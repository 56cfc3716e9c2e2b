// lora_down.cu -- the adapter's down map for the 4-bit matmul with a low-rank
// adapter (QLoRA: "bitsandbytes quantization tutorial" (mljourney.com),
// "QLoRA: Fine-Tuning a 4-bit Model"; "bitsandbytes" (ozercemkelahmet.com),
// "Fine-tuning with adapters on a 4-bit model": r = 16, lora_alpha = 32).
//
//   v[m, j] = fp32(s * sum_k X[m, k] * A[j, k])          (fp32 sum)
//   T[m, j] = bf16_rn(v),  T[m, r + j] = bf16_rn(v - T[m, j])   for j < r
//   T[m, j] = 0                                           for 2r <= j < 64
//
// The bf16 pair (hi, lo) carries v to about 16 significant bits, so the
// adapter term is not rounded to bf16 on its way to the tensor cores.  T is
// stored [m, 64] so the GEMM loads it with the same 64-wide, 128-byte swizzled
// TMA box as an activation stage and adds [hi | lo] . [B | B]^T to its
// accumulator as one more reduction stage.  One CTA per 16 rows of X; 16
// warps split K in 32-wide chunks (four chunks' loads in flight per warp);
// each warp accumulates a 16 x r tile with mma.sync m16n8k16 (bf16 in, fp32
// accumulate); the 16 partial tiles are added in warp order through shared
// memory (deterministic).
#include "nf4_common.cuh"
#include "internal.h"

namespace nf4 {
namespace {

constexpr int kWarps = 16;
constexpr int kTCols = 64;  // row length of T (the stage width of the GEMM)

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// NT = r / 8 column tiles of 8
template <int NT>
__global__ void __launch_bounds__(kWarps * 32) lora_down_kernel(const __nv_bfloat16* __restrict__ x,
                                                                 const __nv_bfloat16* __restrict__ a, int m_total,
                                                                 int cols, float scale, __nv_bfloat16* __restrict__ t) {
  __shared__ float red[kWarps][16][NT * 8];
  // the GEMM that consumes T starts once every CTA is past this wait, i.e. once this launch's own
  // predecessor has finished: the GEMM can then read X and the weight at once and waits for this grid
  // only before its adapter stage loads T
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int m0 = blockIdx.x * 16;
  const bool v0 = m0 + g < m_total, v1 = m0 + g + 8 < m_total;
  const __nv_bfloat16* x0 = x + (int64_t)(v0 ? m0 + g : 0) * cols;
  const __nv_bfloat16* x1 = x + (int64_t)(v1 ? m0 + g + 8 : 0) * cols;
  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
  // Lane (g, q) owns k positions 8q .. 8q+7 of a 32-wide chunk: positions 8q..8q+3 feed the first MMA's
  // fragment slots (2q, 2q+1, 2q+8, 2q+9), 8q+4..8q+7 the second's, for X and A alike (a dot product does
  // not depend on the order of its terms), so each operand row is one 16-byte load.
#pragma unroll 4
  for (int c = warp; c < cols / 32; c += kWarps) {
    const int k = c * 32 + q * 8;
    const uint4 xa = v0 ? __ldg(reinterpret_cast<const uint4*>(x0 + k)) : make_uint4(0, 0, 0, 0);
    const uint4 xb = v1 ? __ldg(reinterpret_cast<const uint4*>(x1 + k)) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(a + (int64_t)(nt * 8 + g) * cols + k));
      mma16816(acc[nt], xa.x, xb.x, xa.y, xb.y, w.x, w.y);
      mma16816(acc[nt], xa.z, xb.z, xa.w, xb.w, w.z, w.w);
    }
  }
  // accumulator fragment: (row g, columns 2q, 2q+1) and (row g+8, the same columns) of each 8-column tile
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    red[warp][g][nt * 8 + 2 * q] = acc[nt][0];
    red[warp][g][nt * 8 + 2 * q + 1] = acc[nt][1];
    red[warp][g + 8][nt * 8 + 2 * q] = acc[nt][2];
    red[warp][g + 8][nt * 8 + 2 * q + 1] = acc[nt][3];
  }
  __syncthreads();
  constexpr int R = NT * 8;
  for (int i = threadIdx.x; i < 16 * kTCols; i += blockDim.x) {
    const int row = i / kTCols, j = i % kTCols;
    if (m0 + row >= m_total) continue;
    __nv_bfloat16 out = __float2bfloat16_rn(0.0f);
    if (j < 2 * R) {
      const int jj = j < R ? j : j - R;
      float sum = 0.0f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) sum += red[w][row][jj];
      const float v = __fmul_rn(scale, sum);
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      out = j < R ? hi : __float2bfloat16_rn(__fsub_rn(v, __bfloat162float(hi)));
    }
    t[(int64_t)(m0 + row) * kTCols + j] = out;
  }
}

}  // namespace

cudaError_t launch_lora_down(const void* x, const void* a, int64_t m, int64_t cols, int r, float scale, void* t,
                             cudaStream_t stream) {
  const dim3 grid((unsigned)((m + 15) / 16));
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  const auto* ab = static_cast<const __nv_bfloat16*>(a);
  auto* tb = static_cast<__nv_bfloat16*>(t);
  const int M = (int)m, C = (int)cols;
  cudaError_t e;
  switch (r) {
    case 16: e = launch_pdl(lora_down_kernel<2>, grid, dim3(kWarps * 32), 0, stream, xb, ab, M, C, scale, tb); break;
    case 32: e = launch_pdl(lora_down_kernel<4>, grid, dim3(kWarps * 32), 0, stream, xb, ab, M, C, scale, tb); break;
    default: return cudaErrorInvalidValue;
  }
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace nf4
