// gemm_sm100.cu -- prefill GEMM Y = X . Wc^T on tcgen05 tensor cores.
//
// "bitsandbytes" (ozercemkelahmet.com/tools), "How it works" Step 5: matrix
// hardware works best on 16-bit numbers, so each NF4 block is expanded back to
// 16-bit (bf16_rn(RN(code[i] * a)), compute dtype bfloat16 per "bitsandbytes
// quantization tutorial", mljourney.com) and then multiplied.  Here the
// expansion happens tile by tile in shared memory, and the multiply is a
// tcgen05 bf16 x bf16 -> fp32 MMA with the accumulator in tensor memory.
//
// Tile: 128 weight rows (UMMA M, operand A) x 256 activation rows (UMMA N,
// operand B) x 64 k per pipeline stage (one level-1 block per weight row).
// D[n, m] lives in TMEM (lane = weight row, column = activation row); two
// accumulators (2 x 256 columns) let the MMA run one tile ahead of the
// epilogue.  One persistent CTA per SM walks the tiles; warp roles:
//   warps 0-3   epilogue: tcgen05.ld -> bf16 -> Y (warp w reads TMEM lanes 32w..)
//   warps 4-11  dequant producers, two groups of four taking alternate stages:
//               thread p decodes weight row p of the stage (64 codes) with the
//               byte-permute tables and writes the 128B-swizzled K-major tile
//   warp 12     TMA producer: activation tile (256 x 64 bf16, 128B swizzle)
//   warp 13     TMEM allocator and MMA issuer (one elected thread)
// Every mbarrier wait is bounded; on timeout the device error word is set and
// the roles leave their loops, so a fault cannot hang the GPU.
#include <cuda.h>

#include "nf4_common.cuh"
#include "nf4_decode.cuh"
#include "internal.h"

namespace nf4 {
namespace {

constexpr int kTileN = 128;       // weight rows per tile (UMMA M)
constexpr int kTileM = 256;       // activation rows per tile (UMMA N)
constexpr int kTileK = 64;        // k per stage (128 bytes of bf16: one swizzle atom)
constexpr int kStages = 4;
constexpr int kABytes = kTileN * kTileK * 2;  // 16 KB
constexpr int kBBytes = kTileM * kTileK * 2;  // 32 KB
constexpr int kAccCols = kTileM;              // fp32 columns per accumulator
constexpr int kTmemCols = 2 * kAccCols;       // 512
constexpr int kThreads = 14 * 32;
constexpr int kEpiWarps = 4;
constexpr int kProdWarp0 = 4;                 // producers: warps 4..11
constexpr int kTmaWarp = 12;
constexpr int kMmaWarp = 13;
constexpr size_t kSmemBytes = (size_t)kStages * (kABytes + kBBytes) + 1024 /*align*/ + 2048 /*barriers, lut*/;

struct Smem {  // placed after the 1024-aligned stage buffers
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
  int abort;
  float unit_lut[256];
};

// ------------------------------------------------------------------ tcgen05 / TMA wrappers

__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  // K-major, 128-byte swizzle: rows of 128 B, 8-row groups 1024 B apart
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fffu);          // start address
  d |= (uint64_t)1 << 16;                          // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;                // stride byte offset: next 8-row group
  d |= (uint64_t)1 << 46;                          // descriptor version (Blackwell)
  d |= (uint64_t)2 << 61;                          // layout: SWIZZLE_128B
  return d;
}

// kind::f16 instruction descriptor: bf16 A and B, fp32 D, both K-major
__host__ __device__ constexpr uint32_t instr_desc(int m, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 consecutive fp32 columns (one register per column) of this warp's subpartition
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ bool aborted(Smem* sm) { return *(volatile int*)&sm->abort != 0; }

// bounded wait; on failure mark the CTA aborted so every role leaves its loop
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Smem* sm, unsigned* err) {
  if (aborted(sm)) return false;
  if (mbar_wait_bounded(bar, parity, err)) return true;
  *(volatile int*)&sm->abort = 1;
  return false;
}

// ------------------------------------------------------------------ kernel

template <bool kDQ>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const uint8_t* __restrict__ packed, Scales s, int rows, int cols, int m_total,
                const __grid_constant__ CUtensorMap xmap, __nv_bfloat16* __restrict__ y, unsigned* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;  // 1024-aligned stage buffers (swizzle atoms)
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t a_smem0 = base, b_smem0 = base + kStages * kABytes;
  uint8_t* a_gen0 = gbase;
  Smem* sm = reinterpret_cast<Smem*>(gbase + kStages * (kABytes + kBBytes));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles_n = rows / kTileN;
  const int ntiles_m = (m_total + kTileM - 1) / kTileM;
  const int ntiles = ntiles_n * ntiles_m;
  const int kstages = cols / kTileK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm->full[i], 4 + 1);  // 4 producer warps + the TMA arrive.expect_tx
      mbar_init(&sm->empty[i], 1);     // tcgen05.commit
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm->acc_full[i], 1);
      mbar_init(&sm->acc_empty[i], kEpiWarps);
    }
    sm->abort = 0;
    fence_mbar_init();
  }
  if (kDQ && threadIdx.x < 256) sm->unit_lut[threadIdx.x] = dq_unit(threadIdx.x, s.dq_code);
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm->tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;

  if (warp >= kProdWarp0 && warp < kTmaWarp) {
    // ------------------------------------------------ dequant producers
    const int group = (warp - kProdWarp0) >> 2;          // 0 or 1: alternate stages
    const int p = ((warp - kProdWarp0) & 3) * 32 + lane;  // weight row within the tile
    const float mu = kDQ ? *s.mean : 0.0f;
    const int64_t rb = cols / kBlock;
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      const int64_t row = (int64_t)(tile / ntiles_m) * kTileN + p;
      for (int ks = 0; ks < kstages; ++ks, ++it) {
        if ((int)(it & 1) != group) continue;
        const int st = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        // issue the global loads before waiting for the stage to drain
        const uint4* src = reinterpret_cast<const uint4*>(packed + row * (cols / 2) + (int64_t)ks * 32);
        const uint4 w0 = __ldg(src), w1 = __ldg(src + 1);
        const int64_t b = row * rb + ks;
        float a;
        if (kDQ)
          a = dq_absmax(sm->unit_lut[s.q[b]], s.scale[b / kDqBlock], mu);
        else
          a = __ldg(s.absmax + b);
        const Table T = make_table(a);
        if (!wait_or_abort(&sm->empty[st], ph ^ 1, sm, err)) break;
        uint8_t* dst = a_gen0 + st * kABytes + p * 128;
        const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t d[4];
          decode_word(words[c], T, d);
          *reinterpret_cast<uint4*>(dst + ((c ^ (p & 7)) << 4)) = make_uint4(d[0], d[1], d[2], d[3]);
        }
        fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->full[st]);
      }
      if (aborted(sm)) break;
    }
  } else if (warp == kTmaWarp) {
    // ------------------------------------------------ activation tiles via TMA
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap)) : "memory");
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < ntiles && !aborted(sm); tile += gridDim.x) {
        const int m0 = (tile % ntiles_m) * kTileM;
        for (int ks = 0; ks < kstages; ++ks, ++it) {
          const int st = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!wait_or_abort(&sm->empty[st], ph ^ 1, sm, err)) break;
          mbar_expect_tx(&sm->full[st], kBBytes);
          tma_load_2d(b_smem0 + st * kBBytes, &xmap, ks * kTileK, m0, &sm->full[st]);
        }
      }
      // drain: wait for the copies still in flight into the stages
      const uint32_t issued = it;
      for (uint32_t j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
        mbar_wait_bounded(&sm->full[j % kStages], (j / kStages) & 1, err);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc(kTileN, kTileM);
      uint32_t it = 0, tcount = 0;
      for (int tile = blockIdx.x; tile < ntiles && !aborted(sm); tile += gridDim.x, ++tcount) {
        const int acc = tcount & 1;
        if (!wait_or_abort(&sm->acc_empty[acc], ((tcount >> 1) & 1) ^ 1, sm, err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * kAccCols;
        bool ok = true;
        for (int ks = 0; ks < kstages; ++ks, ++it) {
          const int st = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          if (!wait_or_abort(&sm->full[st], ph, sm, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = a_smem0 + st * kABytes, b_addr = b_smem0 + st * kBBytes;
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk)  // 16 bf16 = 32 bytes per MMA along k
            tc_mma(d_tmem, smem_desc_sw128(a_addr + kk * 32), smem_desc_sw128(b_addr + kk * 32), idesc,
                   (ks | kk) != 0);
          tc_commit(&sm->empty[st]);  // stage free once these MMAs have read it
        }
        if (!ok) break;
        tc_commit(&sm->acc_full[acc]);  // accumulator ready for the epilogue
      }
    }
  } else if (warp < kEpiWarps) {
    // ------------------------------------------------ epilogue: TMEM -> bf16 -> Y
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tcount) {
      const int acc = tcount & 1;
      if (!wait_or_abort(&sm->acc_full[acc], (tcount >> 1) & 1, sm, err)) break;
      tc_fence_after();
      const int64_t n = (int64_t)(tile / ntiles_m) * kTileN + warp * 32 + lane;
      const int m0 = (tile % ntiles_m) * kTileM;
#pragma unroll 1
      for (int c = 0; c < kTileM / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + acc * kAccCols + c * 32, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int m = m0 + c * 32 + j;
          if (m < m_total) y[(int64_t)m * rows + n] = __float2bfloat16_rn(__uint_as_float(v[j]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm->acc_empty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ------------------------------------------------------------------ host side

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled get_encoder() {
  static EncodeTiled fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  }
  return fn;
}

}  // namespace

size_t gemm_workspace_bytes(int64_t, int64_t, int64_t) { return 0; }

cudaError_t launch_gemm(const uint8_t* packed, const Scales& s, int64_t rows, int64_t cols, const void* x, int64_t m,
                        void* y, void*, unsigned* err, cudaStream_t stream, int num_sms) {
  auto* yb = static_cast<__nv_bfloat16*>(y);
  if (m <= 64) return launch_gemv(packed, s, rows, cols, x, (int)m, y, stream, num_sms);
  if (rows > INT32_MAX || cols > INT32_MAX || m > INT32_MAX) return cudaErrorInvalidValue;
  EncodeTiled encode = get_encoder();
  if (encode == nullptr) return cudaErrorNotSupported;
  CUtensorMap xmap;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)m};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kTileK, (cuuint32_t)kTileM};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int ntiles = (int)((rows / kTileN) * ((m + kTileM - 1) / kTileM));
  const int grid = ntiles < num_sms ? ntiles : num_sms;
  const bool dq = s.absmax == nullptr;
  cudaError_t e;
  if (dq) {
    e = cudaFuncSetAttribute(gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    gemm_kernel<true><<<grid, kThreads, kSmemBytes, stream>>>(packed, s, (int)rows, (int)cols, (int)m, xmap, yb, err);
  } else {
    e = cudaFuncSetAttribute(gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    gemm_kernel<false><<<grid, kThreads, kSmemBytes, stream>>>(packed, s, (int)rows, (int)cols, (int)m, xmap, yb, err);
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace nf4
