// gemv.cu -- decode GEMV (batch 1..8) with on-the-fly 4-bit dequantization, one CTA per 16-row tile.
//
// "bitsandbytes" (ozercemkelahmet.com/tools), "How it works" Step 5: each block
// is expanded back to 16-bit with its scale and the code book, then
// multiplied; compute dtype bfloat16 ("bitsandbytes quantization tutorial",
// mljourney.com, "4-bit Loading with NF4").  So the effective weight is
// Wc = bf16_rn(RN(code[idx] * a)) and y[b, n] = bf16_rn(sum_k Wc[n, k] x[b, k])
// with fp32 accumulation.
//
// Mapping (one CTA = one 16-row tile, 8 warps splitting K; one warp step =
// 16 rows x 256 k):
//   lane (g = lane/4, t = lane%4) owns rows g and g+8 of the tile and level-1
//   block t of the step (64 codes = 32 bytes per row, two 16-byte loads).
//   Per (row, block) the lane builds the 16 bf16 values bf16_rn(code[i] * a)
//   and keeps their low and high bytes as four 8-byte byte-permute pools; a
//   packed 32-bit word of 8 codes is then decoded with byte permutes: the
//   code nibbles themselves are the permute selectors, bit 3 of each nibble
//   picks the pool half.
//   The decoded bf16 pairs are the A operand of mma.sync m16n8k16 (weights
//   as the M side, activations as the N side: batch <= 8 per n-tile), so one
//   decode feeds up to 8 activation rows per n-tile.  Lanes with the same t
//   use the same four k positions per MMA, which keeps the B fragment a
//   contiguous 8-byte slice of x.
// At batch 1 the decode, not HBM, bounds the kernel, so three quarters of it
// leave the ALU pipe: row g+8 and the second half of row g's step are
// expanded through a 64 KB shared table of fp32 code pairs instead (one copy
// per bank; a byte permute of the packed word with the lane's offset is the
// address, then two multiplies by a and one bf16x2 convert) -- the same
// bf16_rn(RN(code * a)) values.  With more
// activation rows the lookups would compete with the activation loads, so
// larger batches decode both rows with byte permutes.
// Partial sums of the 8 warps are added in a fixed order through shared
// memory, so results are deterministic.
// One launch may cover up to four weights that read the same x (q/k/v or
// gate/up of a decoder layer): the grid is the concatenation of their 16-row
// tiles and each CTA picks its weight from the cumulative tile counts, so
// small projections share the GPU with large ones instead of leaving SMs idle.
#include <atomic>

#include "nf4_common.cuh"
#include "nf4_decode.cuh"
#include "internal.h"

namespace nf4 {
namespace {

constexpr int kWarps = 8;
constexpr int kStepK = 256;  // k per warp step (4 level-1 blocks)

// up to kMaxGroup weights sharing cols, the scale kind and the input x; CTA b works on 16-row tile
// b - tile_end[i - 1] of weight i, the first i with b < tile_end[i]
struct GemvGroup {
  const uint8_t* packed[kMaxGroup];
  Scales s[kMaxGroup];
  __nv_bfloat16* y[kMaxGroup];
  int tile_end[kMaxGroup];
  int count;
};
// fp32 code pairs: entry v of copy c at 256 v + 8 c, 16 copies (the first 128 bytes of every 256-byte row; a
// byte permute of the code with the lane's offset is the address).  A 64-bit shared load is served in two
// half-warp phases, so lane l reading copy l % 16 keeps each phase free of bank conflicts.
constexpr int kPairTableBytes = 256 * 32 * 8;

__constant__ float c_code_gemv[2][16] = {NF4_CODE_INIT, FP4_CODE_INIT};  // by code book: NF4, FP4

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

struct StepData {
  uint4 w0[2], w1[2];  // 32 code bytes of row g and of row g+8
  float s0, s1;        // plain scales, or second-level block absmax (double quant)
  uint32_t q0, q1;     // 8-bit scale codes (double quant)
};

template <bool kDQ>
__device__ __forceinline__ void load_step(StepData& d, const uint8_t* __restrict__ packed, const Scales& s,
                                          int64_t row0, int64_t cols, int64_t blk, bool valid) {
  if (!valid) {
    d.w0[0] = d.w0[1] = d.w1[0] = d.w1[1] = make_uint4(0x77777777u, 0x77777777u, 0x77777777u, 0x77777777u);
    d.s0 = d.s1 = 0.0f;
    d.q0 = d.q1 = 0;
    return;
  }
  const int64_t rb = cols / kBlock;  // blocks per row
  const uint4* p0 = reinterpret_cast<const uint4*>(packed + row0 * (cols / 2) + blk * 32);
  const uint4* p1 = reinterpret_cast<const uint4*>(packed + (row0 + 8) * (cols / 2) + blk * 32);
  d.w0[0] = __ldcs(p0);
  d.w0[1] = __ldcs(p0 + 1);
  d.w1[0] = __ldcs(p1);
  d.w1[1] = __ldcs(p1 + 1);
  const int64_t b0 = row0 * rb + blk, b1 = (row0 + 8) * rb + blk;
  if (kDQ) {
    d.q0 = s.q[b0];
    d.q1 = s.q[b1];
    d.s0 = s.scale[b0 / kDqBlock];
    d.s1 = s.scale[b1 / kDqBlock];
  } else {
    d.s0 = __ldcs(s.absmax + b0);
    d.s1 = __ldcs(s.absmax + b1);
  }
}

template <int NT, bool kDQ, bool kTable, int kBook>
__global__ void __launch_bounds__(kWarps * 32, NT >= 4 ? 1 : 2)
    gemv_kernel(GemvGroup grp, int64_t cols, const __nv_bfloat16* __restrict__ x, int batch) {
  __shared__ float unit_lut[kDQ ? 256 : 1];
  __shared__ float red[kWarps][16][8 * NT];
  extern __shared__ __align__(16) uint8_t pair_table[];  // entry v of lane l at 256 v + 8 (l % 16)
  pdl_launch_dependents();
  // this CTA's weight of the group (every index below is a compile-time constant)
  const uint8_t* __restrict__ packed = grp.packed[0];
  Scales s = grp.s[0];
  __nv_bfloat16* __restrict__ y = grp.y[0];
  int tile0 = 0, tile1 = grp.tile_end[0];
#pragma unroll
  for (int i = 1; i < kMaxGroup; ++i)
    if (i < grp.count && (int)blockIdx.x >= grp.tile_end[i - 1]) {
      packed = grp.packed[i];
      s = grp.s[i];
      y = grp.y[i];
      tile0 = grp.tile_end[i - 1];
      tile1 = grp.tile_end[i];
    }
  const int tile = (int)blockIdx.x - tile0;
  const int64_t rows = (int64_t)(tile1 - tile0) * 16;
  if (kDQ) unit_lut[threadIdx.x & 255] = dq_unit(threadIdx.x & 255, s.dq_code);
  if (kTable) {
    // the 16 levels through shared memory first: the table's lanes read them at different indices, which a
    // constant-memory read would serialise
    __shared__ float code_s[16];
    if (threadIdx.x < 16) code_s[threadIdx.x] = c_code_gemv[kBook][threadIdx.x];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 256 * 8 / (kWarps * 32); ++k) {
      const int idx = threadIdx.x + k * kWarps * 32;  // 16-byte pieces: copies 2i, 2i + 1 of one entry
      const int v = idx >> 3, i = idx & 7;
      const float hi = code_s[v >> 4], lo = code_s[v & 15];
      *reinterpret_cast<float4*>(pair_table + v * 256 + i * 16) = make_float4(hi, lo, hi, lo);
    }
  }
  __syncthreads();
  pdl_wait();
  const float mu = kDQ ? *s.mean : 0.0f;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int64_t row0 = (int64_t)tile * 16 + g;
  const int64_t nblk = cols / kBlock;
  const int64_t nsteps = (cols + kStepK - 1) / kStepK;

  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[nt][j] = 0.0f;

  // activation rows fed by this lane, one per n-tile (null: padding row)
  const __nv_bfloat16* xrow[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) xrow[nt] = (8 * nt + g < batch) ? x + (int64_t)(8 * nt + g) * cols : nullptr;

  const DecodeMul dm = decode_mul();
  const uint32_t lane8 = (uint32_t)((lane & 15) * 8);
  StepData cur, nxt;
  int64_t st = warp;
  if (st < nsteps) load_step<kDQ>(cur, packed, s, row0, cols, st * 4 + t, st * 4 + t < nblk);
  for (; st < nsteps; st += kWarps) {
    const int64_t blk = st * 4 + t;
    const bool valid = blk < nblk;
    if (st + kWarps < nsteps) load_step<kDQ>(nxt, packed, s, row0, cols, (st + kWarps) * 4 + t, (st + kWarps) * 4 + t < nblk);
    float a0 = cur.s0, a1 = cur.s1;
    if (kDQ) {
      a0 = dq_absmax(unit_lut[cur.q0], cur.s0, mu);
      a1 = dq_absmax(unit_lut[cur.q1], cur.s1, mu);
    }
    const Table T0 = make_table<kBook>(a0);
    Table T1;
    if (!kTable) T1 = make_table<kBook>(a1);
    const uint32_t w0[8] = {cur.w0[0].x, cur.w0[0].y, cur.w0[0].z, cur.w0[0].w,
                            cur.w0[1].x, cur.w0[1].y, cur.w0[1].z, cur.w0[1].w};
    const uint32_t w1[8] = {cur.w1[0].x, cur.w1[0].y, cur.w1[0].z, cur.w1[0].w,
                            cur.w1[1].x, cur.w1[1].y, cur.w1[1].z, cur.w1[1].w};
    const int64_t kbase = blk * kBlock;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      // byte-permute pools (ALU pipe), or (kTable) the shared pair table: a byte permute forms the address of
      // this lane's copy, two multiplies and one convert give the pair -- moving decode work off the ALU pipe
      uint32_t d0[4], d1[4];
      if (kTable && j >= 4) {  // (kTable) row g's second half through the table as well
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const float2 c = *reinterpret_cast<const float2*>(pair_table + prmt(w0[j], lane8, 0x5504u | (b << 4)));
          d0[b] = pack_bf16x2(__fmul_rn(c.x, a0), __fmul_rn(c.y, a0));
        }
      } else {
        decode_word(w0[j], T0, d0, dm);
      }
      if (kTable) {
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const float2 c = *reinterpret_cast<const float2*>(pair_table + prmt(w1[j], lane8, 0x5504u | (b << 4)));
          d1[b] = pack_bf16x2(__fmul_rn(c.x, a1), __fmul_rn(c.y, a1));
        }
      } else {
        decode_word(w1[j], T1, d1, dm);
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        uint4 xv = make_uint4(0, 0, 0, 0);
        if (xrow[nt] != nullptr && valid) xv = __ldg(reinterpret_cast<const uint4*>(xrow[nt] + kbase + 8 * j));
        // k positions 8j..8j+3: A = (row g: d0[0], d0[1]; row g+8: d1[0], d1[1])
        const uint32_t alo[4] = {d0[0], d1[0], d0[1], d1[1]};
        mma_bf16(acc[nt], alo, xv.x, xv.y);
        const uint32_t ahi[4] = {d0[2], d1[2], d0[3], d1[3]};
        mma_bf16(acc[nt], ahi, xv.z, xv.w);
      }
    }
    cur = nxt;
  }

  // accumulator fragment: c0 (row g, col 2t), c1 (g, 2t+1), c2 (g+8, 2t), c3 (g+8, 2t+1)
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    red[warp][g][8 * nt + 2 * t] = acc[nt][0];
    red[warp][g][8 * nt + 2 * t + 1] = acc[nt][1];
    red[warp][g + 8][8 * nt + 2 * t] = acc[nt][2];
    red[warp][g + 8][8 * nt + 2 * t + 1] = acc[nt][3];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 16 * batch; i += blockDim.x) {
    const int r = i & 15, b = i >> 4;
    float sum = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) sum += red[w][r][b];
    y[(int64_t)b * rows + (int64_t)tile * 16 + r] = __float2bfloat16_rn(sum);
  }
}

template <int NT, int kBook>
cudaError_t launch_nt(const GemvGroup& grp, int64_t cols, const void* x, int batch, bool dq, cudaStream_t stream) {
  const unsigned grid = (unsigned)grp.tile_end[grp.count - 1];
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  cudaError_t e = cudaSuccess;
  bool table = false;
  if constexpr (NT == 1) table = batch == 1;  // decode at batch 1: the mixed decode with the 64 KB pair table
  if constexpr (NT == 1) {
    if (table) {
      // the table needs the shared-memory opt-in: set it once per device and variant
      static std::atomic<uint64_t> attr_done[2];
      int dev = 0;
      if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
      if (!(attr_done[dq].load() & (1ull << dev))) {
        e = cudaFuncSetAttribute(
            dq ? (const void*)gemv_kernel<NT, true, true, kBook> : (const void*)gemv_kernel<NT, false, true, kBook>,
            cudaFuncAttributeMaxDynamicSharedMemorySize, kPairTableBytes);
        if (e != cudaSuccess) return e;
        attr_done[dq].fetch_or(1ull << dev);
      }
      e = dq ? launch_pdl(gemv_kernel<NT, true, true, kBook>, dim3(grid), dim3(kWarps * 32), kPairTableBytes, stream,
                          grp, cols, xb, batch)
             : launch_pdl(gemv_kernel<NT, false, true, kBook>, dim3(grid), dim3(kWarps * 32), kPairTableBytes, stream,
                          grp, cols, xb, batch);
    }
  }
  if (!table)
    e = dq ? launch_pdl(gemv_kernel<NT, true, false, kBook>, dim3(grid), dim3(kWarps * 32), 0, stream, grp, cols, xb, batch)
           : launch_pdl(gemv_kernel<NT, false, false, kBook>, dim3(grid), dim3(kWarps * 32), 0, stream, grp, cols, xb,
                        batch);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int kBook>
cudaError_t launch_book(const GemvGroup& grp, int64_t cols, const void* x, int batch, bool dq, cudaStream_t stream) {
  if (batch > 8) return cudaErrorInvalidValue;  // one n-tile of 8 activation rows
  return launch_nt<1, kBook>(grp, cols, x, batch, dq, stream);
}

cudaError_t launch_group(const GemvGroup& grp, int64_t cols, const void* x, int batch, bool dq,
                         cudaStream_t stream) {
  return grp.s[0].book ? launch_book<1>(grp, cols, x, batch, dq, stream) : launch_book<0>(grp, cols, x, batch, dq, stream);
}

}  // namespace

// batch <= 8: one n-tile of the mma holds every activation row
cudaError_t launch_gemv(const uint8_t* packed, const Scales& s, int64_t rows, int64_t cols, const void* x, int batch,
                        void* y, unsigned* err, cudaStream_t stream, int num_sms) {
  (void)err;
  (void)num_sms;
  if (rows / 16 > INT32_MAX) return cudaErrorInvalidValue;
  GemvGroup grp = {};
  grp.packed[0] = packed;
  grp.s[0] = s;
  grp.y[0] = static_cast<__nv_bfloat16*>(y);
  grp.tile_end[0] = (int)(rows / 16);
  grp.count = 1;
  return launch_group(grp, cols, x, batch, s.absmax == nullptr, stream);
}

// several weights with the same cols and scale kind, one input x: one launch whose CTAs cover the 16-row
// tiles of every weight in turn
cudaError_t launch_gemv_group(const uint8_t* const* packed, const Scales* s, const int64_t* rows, int count,
                              int64_t cols, const void* x, int batch, void* const* y, unsigned* err,
                              cudaStream_t stream, int num_sms) {
  if (count < 1 || count > kMaxGroup) return cudaErrorInvalidValue;
  (void)err;
  (void)num_sms;
  GemvGroup grp = {};
  int64_t tiles = 0;
  for (int i = 0; i < count; ++i) {
    tiles += rows[i] / 16;
    if (tiles > INT32_MAX) return cudaErrorInvalidValue;
    grp.packed[i] = packed[i];
    grp.s[i] = s[i];
    grp.y[i] = static_cast<__nv_bfloat16*>(y[i]);
    grp.tile_end[i] = (int)tiles;
  }
  grp.count = count;
  return launch_group(grp, cols, x, batch, s[0].absmax == nullptr, stream);
}

}  // namespace nf4
