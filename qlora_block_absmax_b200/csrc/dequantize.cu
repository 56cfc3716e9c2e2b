// dequantize.cu -- NF4 (and FP4) dequantization.
//
// "bitsandbytes" (ozercemkelahmet.com/tools), "How it works" Step 5: a block is
// expanded back with its scale and the code book: w^ = RN(code[idx] * a).
// With double quantization ("Double quantization") the scale is rebuilt first:
// a^ = RN(RN(unit(q) * m) + mu), unit(q) = RN(dec(q) / Q).
//
// Level-1 blocks of 32, 64, 128 or 256 elements.  fp32 output: 2 to 16 lanes
// own one block (16 elements each: one 8-byte load of packed codes); codes are
// looked up in a 16-entry shared table, multiplied by the block scale and
// written with 16-byte streaming stores.  bf16 output: one lane per 64-element
// chunk, its scale that of the block holding it (two scales for 32-blocks).
#include "nf4_common.cuh"
#include "nf4_decode.cuh"
#include "internal.h"

namespace nf4 {
namespace {

__constant__ float c_code[2][16] = {NF4_CODE_INIT, FP4_CODE_INIT};  // by code book: NF4, FP4
// bf16 output: warps per CTA.  Four (up to 16 CTAs per SM) measured 1 % faster than eight at 4096x4096 and 17 %
// at 1024x1024: the last partial wave of CTAs is smaller.
constexpr int kDeqWarps = 4;

template <bool kDQ>
__device__ __forceinline__ float block_scale(const Scales& s, const float* unit_lut, int64_t b) {
  if (!kDQ) return s.absmax[b];
  return dq_absmax(unit_lut[s.q[b]], s.scale[b / kDqBlock], *s.mean);
}

template <bool kDQ, bool kBF16, int kBook, int kL>
__global__ void __launch_bounds__(256) dequantize_kernel(const uint8_t* __restrict__ packed, Scales s, int64_t n,
                                                         void* __restrict__ out) {
  pdl_launch_dependents();
  __shared__ float code[16];
  __shared__ float unit_lut[kDQ ? 256 : 1];
  if (threadIdx.x < 16) code[threadIdx.x] = c_code[kBook][threadIdx.x];
  if (kDQ) unit_lut[threadIdx.x & 255] = dq_unit(threadIdx.x & 255, s.dq_code);
  __syncthreads();
  pdl_wait();

  // kL lanes per block of kB = 16 kL elements, 16 elements (8 code bytes) each
  constexpr int kB = 16 * kL;
  const int sub = threadIdx.x & (kL - 1);
  const int64_t nfull = n / kB;
  const int64_t nblocks = (n + kB - 1) / kB;
  const int64_t groups = (int64_t)gridDim.x * (blockDim.x / kL);
  const int64_t gid = (int64_t)blockIdx.x * (blockDim.x / kL) + threadIdx.x / kL;
  constexpr int kUnroll = 4;  // blocks per group per iteration: four loads in flight per lane

  for (int64_t b0 = gid; b0 < nblocks; b0 += groups * kUnroll) {
    uint2 pk[kUnroll];
    float a[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {  // issue every load first
      const int64_t b = b0 + u * groups;
      pk[u] = (b < nfull) ? __ldcs(reinterpret_cast<const uint2*>(packed + b * (kB / 2) + sub * 8))
                          : make_uint2(0, 0);
      a[u] = (b < nblocks) ? block_scale<kDQ>(s, unit_lut, b) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t b = b0 + u * groups;
      if (b >= nblocks) break;
      const int64_t first = b * kB + sub * 16;
      if (b < nfull) {
        float v[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t lo = (pk[u].x >> (8 * j)) & 0xffu, hi = (pk[u].y >> (8 * j)) & 0xffu;
          v[2 * j] = __fmul_rn(code[lo >> 4], a[u]);
          v[2 * j + 1] = __fmul_rn(code[lo & 15], a[u]);
          v[8 + 2 * j] = __fmul_rn(code[hi >> 4], a[u]);
          v[8 + 2 * j + 1] = __fmul_rn(code[hi & 15], a[u]);
        }
        if (kBF16) {
          uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + first);
          __stcs(o, make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                               pack_bf16x2(v[6], v[7])));
          __stcs(o + 1, make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                                   pack_bf16x2(v[14], v[15])));
        } else {
          float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + first);
#pragma unroll
          for (int j = 0; j < 4; ++j) __stcs(o + j, make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
        }
      } else {
#pragma unroll 1
        for (int i = 0; i < 16; ++i) {
          const int64_t e = first + i;
          if (e >= n) break;
          const uint8_t byte = packed[e / 2];
          const float v = __fmul_rn(code[(e & 1) ? (byte & 15) : (byte >> 4)], a[u]);
          if (kBF16)
            static_cast<uint16_t*>(out)[e] = (uint16_t)(pack_bf16x2(v, 0.0f) & 0xffffu);
          else
            static_cast<float*>(out)[e] = v;
        }
      }
    }
  }
}

// bf16 output: one lane per 64-element chunk.  The lane builds the chunk's 16
// bf16 values bf16_rn(RN(code[i] * a)) as byte-permute pools (the same decode
// the matmuls use) and expands its 32 code bytes with byte permutes.  The
// warp's 32 consecutive blocks (4 KB of bf16) go through a swizzled shared
// tile so the global stores are 512 contiguous bytes per instruction.
template <bool kDQ, int kBook, int kB>
__global__ void __launch_bounds__(kDeqWarps * 32) dequantize_bf16_kernel(const uint8_t* __restrict__ packed, Scales s,
                                                              int64_t n, __nv_bfloat16* __restrict__ out) {
  __shared__ float unit_lut[kDQ ? 256 : 1];
  __shared__ __align__(16) uint4 stage[kDeqWarps][32 * 8];  // per warp: 32 chunks x 8 pieces of 16 bytes
  pdl_launch_dependents();
  if (kDQ)
    for (int i = threadIdx.x; i < 256; i += blockDim.x) unit_lut[i] = dq_unit(i, s.dq_code);
  __syncthreads();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const DecodeMul dm = decode_mul();
  uint4* st = stage[warp];
  const int64_t nfull = n / kBlock;
  const int64_t nblocks = (n + kBlock - 1) / kBlock;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t b0 = ((int64_t)blockIdx.x * (blockDim.x >> 5) + warp) * 32; b0 < nblocks; b0 += nwarps * 32) {
    const int64_t b = b0 + lane;
    const bool full_warp = b0 + 32 <= nfull;  // all 32 blocks complete: the coalesced path
    if (full_warp) {
      const uint4* src = reinterpret_cast<const uint4*>(packed + b * (kBlock / 2));
      const uint4 w0 = __ldcs(src), w1 = __ldcs(src + 1);
      // the chunk's scale: its block (kB >= 64), or one per half (kB = 32: words 0-3 and 4-7)
      const Table T = make_table<kBook>(block_scale<kDQ>(s, unit_lut, kB >= 64 ? b / (kB / 64) : 2 * b));
      Table T2;
      if (kB == 32) T2 = make_table<kBook>(block_scale<kDQ>(s, unit_lut, 2 * b + 1));
      const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t d[4];
        decode_word(words[c], (kB == 32 && c >= 4) ? T2 : T, d, dm);
        st[lane * 8 + (c ^ (lane & 7))] = make_uint4(d[0], d[1], d[2], d[3]);  // XOR swizzle: no bank conflicts
      }
      __syncwarp();
      uint4* o = reinterpret_cast<uint4*>(out + b0 * kBlock);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int piece = i * 32 + lane;  // 16-byte piece of the warp's 4 KB
        const int blk = piece >> 3, c = piece & 7;
        __stcs(o + piece, st[blk * 8 + (c ^ (blk & 7))]);
      }
      __syncwarp();
    } else if (b < nblocks) {
      const Table T = make_table<kBook>(block_scale<kDQ>(s, unit_lut, kB >= 64 ? b / (kB / 64) : 2 * b));
      Table T2;
      const bool two = kB == 32 && 2 * b + 1 < (n + kB - 1) / kB;  // a second 32-block in this chunk
      if (kB == 32 && two) T2 = make_table<kBook>(block_scale<kDQ>(s, unit_lut, 2 * b + 1));
      if (b < nfull) {
        const uint4* src = reinterpret_cast<const uint4*>(packed + b * (kBlock / 2));
        const uint4 w0 = __ldcs(src), w1 = __ldcs(src + 1);
        const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        uint4* o = reinterpret_cast<uint4*>(out + b * kBlock);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t d[4];
          decode_word(words[c], (kB == 32 && c >= 4) ? T2 : T, d, dm);
          __stcs(o + c, make_uint4(d[0], d[1], d[2], d[3]));
        }
      } else {
        // short last chunk: element by element from its block's table
        for (int64_t e = b * kBlock; e < n; ++e) {
          const uint8_t byte = packed[e / 2];
          const uint32_t nib = (e & 1) ? (byte & 15u) : (byte >> 4);
          uint32_t d[4];
          decode_word(nib * 0x11111111u, (kB == 32 && e - b * kBlock >= 32) ? T2 : T, d);  // every nibble: this code
          reinterpret_cast<uint16_t*>(out)[e] = (uint16_t)(d[0] & 0xffffu);
        }
      }
    }
  }
}

template <int kBook, int kB>
cudaError_t launch_block(const uint8_t* packed, const Scales& s, int64_t n, void* out, bool out_bf16,
                         cudaStream_t stream, int num_sms) {
  const int64_t cap = (int64_t)num_sms * 8;
  const bool dq = s.absmax == nullptr;
  cudaError_t e;
  if (out_bf16) {
    int64_t g2 = ((n + kBlock - 1) / kBlock + 32 * kDeqWarps - 1) / (32 * kDeqWarps);  // 32 chunks of 64 per warp
    if (g2 > 2 * cap) g2 = 2 * cap;
    if (g2 < 1) g2 = 1;
    auto* ob = static_cast<__nv_bfloat16*>(out);
    e = dq ? launch_pdl(dequantize_bf16_kernel<true, kBook, kB>, dim3((unsigned)g2), dim3(kDeqWarps * 32), 0, stream, packed, s, n,
                        ob)
           : launch_pdl(dequantize_bf16_kernel<false, kBook, kB>, dim3((unsigned)g2), dim3(kDeqWarps * 32), 0, stream, packed, s,
                        n, ob);
  } else {
    constexpr int kL = kB / 16;
    int64_t grid = ((n + kB - 1) / kB + 256 / kL - 1) / (256 / kL);
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    const dim3 g((unsigned)grid), b(256);
    e = dq ? launch_pdl(dequantize_kernel<true, false, kBook, kL>, g, b, 0, stream, packed, s, n, out)
           : launch_pdl(dequantize_kernel<false, false, kBook, kL>, g, b, 0, stream, packed, s, n, out);
  }
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int kBook>
cudaError_t launch_book(const uint8_t* packed, const Scales& s, int64_t n, int blocksize, void* out, bool out_bf16,
                        cudaStream_t stream, int num_sms) {
  switch (blocksize) {
    case 32: return launch_block<kBook, 32>(packed, s, n, out, out_bf16, stream, num_sms);
    case 64: return launch_block<kBook, 64>(packed, s, n, out, out_bf16, stream, num_sms);
    case 128: return launch_block<kBook, 128>(packed, s, n, out, out_bf16, stream, num_sms);
    case 256: return launch_block<kBook, 256>(packed, s, n, out, out_bf16, stream, num_sms);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_dequantize(const uint8_t* packed, const Scales& s, int64_t n, int blocksize, void* out,
                              bool out_bf16, cudaStream_t stream, int num_sms) {
  return s.book ? launch_book<1>(packed, s, n, blocksize, out, out_bf16, stream, num_sms)
                : launch_book<0>(packed, s, n, blocksize, out, out_bf16, stream, num_sms);
}

}  // namespace nf4
