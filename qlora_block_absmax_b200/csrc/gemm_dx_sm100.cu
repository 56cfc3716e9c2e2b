// gemm_dx_sm100.cu -- input gradient of the 4-bit matmul, dX = dY . Wc, on
// tcgen05 tensor cores.
//
// "bitsandbytes" (ozercemkelahmet.com/tools), "Strengths and limitations"
// (Limitations), and "bitsandbytes quantization tutorial" (mljourney.com),
// "QLoRA: Fine-Tuning a 4-bit Model": the 4-bit base weight is frozen and gets
// no gradient of its own, but the loss gradient passes through it to the
// adapters and the layers below.  For y = x . Wc^T that is
//   dX[m, k] = bf16_rn( sum_n dY[m, n] * Wc[n, k] ),  Wc = bf16_rn(code * a^),
// the same 16-bit expanded weight as the forward product ("How it works"
// Step 5), accumulated in fp32.
//
// The packed weight is read in its stored [N, K] order: a stage takes 64
// weight rows n (the reduction) x 128 columns k (the output tile).  Producer
// thread p decodes one level-1 block (row n, 64 consecutive k) and writes it as
// one 128-byte row of an MN-major, 128-byte-swizzled shared-memory tile, so
// the MMA reads the transposed operand without any transpose pass:
//   A = Wc^T tile   [128 k (UMMA M, MN-major)] x [64 n]   shared memory
//   B = dY tile     [256 m (UMMA N)]           x [64 n]   shared memory (TMA, K-major)
//   D = dX^T tile   TMEM lane = k, column = m (fp32), two accumulators
// Warp roles (one persistent CTA per SM):
//   warps 0-3   epilogue: tcgen05.ld -> bf16 -> dX (shared with the forward GEMM)
//   warps 4-11  dequant producers, two groups of four taking alternate stages
//   warp 12     TMA producer: dY tile (256 x 64 bf16, 128B swizzle)
//   warp 13     TMEM allocator and MMA issuer (one elected thread)
//   warp 14     TMA producer: packed codes (two 32-byte boxes per row) and scale chunks
// Every mbarrier wait is bounded; on timeout the device error word is set and
// the roles leave their loops.
#include <cuda.h>

#include <atomic>

#include "nf4_common.cuh"
#include "nf4_decode.cuh"
#include "internal.h"
#include "umma.cuh"

namespace nf4 {
namespace {

using namespace umma;

constexpr int kTileR = 64;                     // weight rows (reduction) per stage
// operand ring: stage s holds a dY tile (TMA) and a decoded Wc^T tile (producer warps) that fill and empty
// together, one full and one empty barrier per stage for the single MMA-issuing thread
constexpr int kStages = 4;
constexpr int kWStages = 4;                    // packed-code + scale ring (4 + 4 stages: 223 KB of shared memory)
constexpr int kBBytes = kTileM * kTileR * 2;   // 32 KB: dY tile (operand B)
constexpr int kABytes = kTileR * kTileN * 2;   // 16 KB: decoded tile (operand A)
constexpr int kWHalf = kTileR * 32;            // 2 KB: one level-1 block of codes per row
constexpr int kWBytes = 2 * kWHalf;            // 4 KB: the stage's two blocks per row
constexpr int kSBytes = kTileR * 16;           // 1 KB: 16-byte scale chunk per row
constexpr int kRingBytes = kStages * (kBBytes + kABytes) + kWStages * (kWBytes + kSBytes);
static_assert(kStages * kBBytes >= split_stage_bytes(kTileM), "split reduction staging fits in the operand ring");
constexpr int kTmemCols = 2 * kAccCols;        // two accumulators
constexpr int kThreads = 15 * 32;
constexpr int kProdWarp0 = 4;
constexpr int kTmaWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kTmaWWarp = 14;
constexpr size_t kSmemBytes = (size_t)kRingBytes + kEpiWarps * kStageOutBytes + 1024 /*align*/ +
                              2048 /*barriers, lut*/;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

// A-tile layout (MN-major, 128-byte swizzle): reduction row r, column e (k) at
//   (r / 8) * kKGroup + (e / 64) * kMnAtom + (r % 8) * 128 + (((e % 64) / 8) ^ (r % 8)) * 16 + (e % 8) * 2
constexpr uint32_t kMnAtom = 1024;  // the two 64-column swizzle atoms of an 8-row group sit side by side
constexpr uint32_t kKGroup = 2048;  // 8-row groups along the reduction
static_assert(kTileR / 8 * kKGroup == kABytes && 2 * kMnAtom == kKGroup, "A tile layout");

struct Smem {
  uint64_t wfull[kWStages];
  uint64_t wempty[kWStages];
  uint64_t full[kStages];   // dY tile landed (TMA) and decoded tile written (producer warps)
  uint64_t empty[kStages];  // both consumed by the stage's MMAs (tcgen05.commit)
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
  int abort;
  float unit_lut[256];
};

template <bool kDQ, bool kScaleTma, int kBook>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_dx_kernel(Scales s, int rows, int cols, int m_total, int splits, const __grid_constant__ CUtensorMap ymap,
                   const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                   __nv_bfloat16* __restrict__ dx, float* __restrict__ part, unsigned* __restrict__ tile_count,
                   unsigned* err) {
  extern __shared__ uint8_t smem_raw[];
  pdl_launch_dependents();
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;  // 1024-aligned stage buffers (swizzle atoms)
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t b_smem0 = base;
  const uint32_t a_smem0 = b_smem0 + kStages * kBBytes;
  const uint32_t w_smem0 = a_smem0 + kStages * kABytes;
  const uint32_t s_smem0 = w_smem0 + kWStages * kWBytes;
  uint8_t* a_gen0 = gbase + (a_smem0 - base);
  const uint8_t* w_gen0 = gbase + (w_smem0 - base);
  const uint8_t* s_gen0 = gbase + (s_smem0 - base);
  uint16_t* out_stage = reinterpret_cast<uint16_t*>(gbase + kRingBytes);
  Smem* sm = reinterpret_cast<Smem*>(gbase + kRingBytes + kEpiWarps * kStageOutBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Work wk;
  wk.ntiles_m = (m_total + kTileM - 1) / kTileM;
  wk.tm = kTileM;
  wk.splits = splits;
  wk.units = (cols / kTileN) * wk.ntiles_m * splits;
  wk.kps = rows / kTileR / splits;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kWStages; ++i) {
      mbar_init(&sm->wfull[i], 1);
      mbar_init(&sm->wempty[i], 4);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm->full[i], 1 + 4);  // TMA arrive.expect_tx + the 4 producer warps of the stage's group
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
  pdl_wait();
  const uint32_t tmem = sm->tmem_base;

  if (warp >= kProdWarp0 && warp < kTmaWarp) {
    // ------------------------------------------------ dequant producers
    const int group = (warp - kProdWarp0) >> 2;            // 0 or 1: alternate stages
    const int p = ((warp - kProdWarp0) & 3) * 32 + lane;   // 0..127
    const int r = p & (kTileR - 1);                        // weight row within the stage
    const int h = p >> 6;                                  // which 64-column half of the output tile
    const float mu = kDQ ? *s.mean : 0.0f;
    const int64_t rb = cols / kBlock;
    const DecodeMul dm = decode_mul();
    // this thread's 128-byte row of the A tile: 8-row group, swizzle atom, row within the atom
    const uint32_t a_row = (uint32_t)(r >> 3) * kKGroup + (uint32_t)h * kMnAtom + (uint32_t)(r & 7) * 128u;
    const uint32_t swz = (uint32_t)(r & 7);
    uint32_t it = 0;
    for (int u = blockIdx.x; u < wk.units; u += gridDim.x) {
      const int kb = wk.n0(u) / kBlock + h;  // level-1 block column of this thread's 64 k
      const int ks0 = wk.split(u) * wk.kps;
      for (int ks = ks0; ks < ks0 + wk.kps; ++ks, ++it) {
        if ((int)(it & 1) != group) continue;
        const int ws = it % kWStages, as = it % kStages;
        const uint32_t wph = (it / kWStages) & 1, aph = (it / kStages) & 1;
        if (!wait_or_abort(&sm->wfull[ws], wph, sm, err)) break;
        const uint4* wsrc = reinterpret_cast<const uint4*>(w_gen0 + ws * kWBytes + h * kWHalf + r * 32);
        const uint4 w0 = wsrc[0], w1 = wsrc[1];
        const uint8_t* sc = s_gen0 + ws * kSBytes + r * 16;
        const int64_t n = (int64_t)ks * kTileR + r;
        const int64_t b = n * rb + kb;
        const uint32_t qcode = kDQ && kScaleTma ? sc[kb & 15] : 0u;
        const float plain = !kDQ && kScaleTma ? reinterpret_cast<const float*>(sc)[kb & 3] : 0.0f;
        fence_proxy_async_smem();  // the slot is refilled by TMA after these reads
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->wempty[ws]);
        float a;
        if (kDQ)
          a = dq_absmax(sm->unit_lut[kScaleTma ? qcode : s.q[b]], __ldg(s.scale + b / kDqBlock), mu);
        else
          a = kScaleTma ? plain : __ldg(s.absmax + b);
        const Table T = make_table<kBook>(a);
        const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        uint32_t q[32];  // q[j] = columns 2j, 2j+1 of this row as bf16x2
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t d[4];
          decode_word(words[c], T, d, dm);
          q[4 * c] = d[0];
          q[4 * c + 1] = d[1];
          q[4 * c + 2] = d[2];
          q[4 * c + 3] = d[3];
        }
        if (!wait_or_abort(&sm->empty[as], aph ^ 1, sm, err)) break;  // the MMAs left this slot
        uint8_t* arow = a_gen0 + as * kABytes + a_row;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(arow + (((uint32_t)c ^ swz) << 4)) =
              make_uint4(q[4 * c], q[4 * c + 1], q[4 * c + 2], q[4 * c + 3]);
        fence_proxy_async_smem();  // generic-proxy writes, read by the tensor cores (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->full[as]);
      }
      if (aborted(sm)) break;
    }
  } else if (warp == kTmaWarp) {
    // ------------------------------------------------ TMA: dY tiles
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&ymap)) : "memory");
      uint32_t it = 0;
      for (int u = blockIdx.x; u < wk.units && !aborted(sm); u += gridDim.x) {
        const int ks0 = wk.split(u) * wk.kps;
        const int m0 = wk.m0(u);
        for (int ks = ks0; ks < ks0 + wk.kps; ++ks, ++it) {
          const int xs = it % kStages;
          if (!wait_or_abort(&sm->empty[xs], ((it / kStages) & 1) ^ 1, sm, err)) break;
          mbar_expect_tx(&sm->full[xs], kBBytes);
          tma_load_2d(b_smem0 + xs * kBBytes, &ymap, ks * kTileR, m0, &sm->full[xs]);
        }
      }
      const uint32_t issued = it;  // drain the copies still in flight
      // (a stage's phase also needs the producers' arrivals: after an abort one timed-out wait is enough, the
      // copies have long landed by then)
      for (uint32_t j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
        if (!mbar_wait_bounded(&sm->full[j % kStages], (j / kStages) & 1, err)) break;
    }
  } else if (warp == kTmaWWarp) {
    // ------------------------------------------------ TMA: packed codes and scale chunks
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&wmap)) : "memory");
      if (kScaleTma) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&smap)) : "memory");
      uint32_t it = 0;
      for (int u = blockIdx.x; u < wk.units && !aborted(sm); u += gridDim.x) {
        const int ks0 = wk.split(u) * wk.kps;
        const int k0 = wk.n0(u), kb0 = k0 / kBlock;
        for (int ks = ks0; ks < ks0 + wk.kps; ++ks, ++it) {
          const int ws = it % kWStages;
          if (!wait_or_abort(&sm->wempty[ws], ((it / kWStages) & 1) ^ 1, sm, err)) break;
          mbar_expect_tx(&sm->wfull[ws], kWBytes + (kScaleTma ? kSBytes : 0));
          // codes of columns k0 .. k0+63 and k0+64 .. k0+127 of rows ks*64 .. +63 (32 bytes each)
          tma_load_2d(w_smem0 + ws * kWBytes, &wmap, k0 / 2, ks * kTileR, &sm->wfull[ws]);
          tma_load_2d(w_smem0 + ws * kWBytes + kWHalf, &wmap, k0 / 2 + 32, ks * kTileR, &sm->wfull[ws]);
          // the 16-byte scale chunk holding block columns kb0 and kb0 + 1 (kb0 is even)
          if (kScaleTma)
            tma_load_2d(s_smem0 + ws * kSBytes, &smap, kDQ ? (kb0 & ~15) : (kb0 & ~3), ks * kTileR, &sm->wfull[ws]);
        }
      }
      const uint32_t issued = it;
      for (uint32_t j = (issued > kWStages ? issued - kWStages : 0); j < issued; ++j)
        mbar_wait_bounded(&sm->wfull[j % kWStages], (j / kWStages) & 1, err);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc(kTileN, kTileM, /*a_mn=*/true);
      uint32_t it = 0, ucount = 0;
      for (int u = blockIdx.x; u < wk.units && !aborted(sm); u += gridDim.x, ++ucount) {
        const int acc = ucount & 1;
        if (!wait_or_abort(&sm->acc_empty[acc], ((ucount >> 1) & 1) ^ 1, sm, err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * kAccCols;
        bool ok = true;
        for (int j = 0; j < wk.kps; ++j, ++it) {
          const int st = it % kStages;
          if (!wait_or_abort(&sm->full[st], (it / kStages) & 1, sm, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = a_smem0 + st * kABytes, b_addr = b_smem0 + st * kBBytes;
#pragma unroll
          for (int kk = 0; kk < kTileR / 16; ++kk)  // 16 weight rows per MMA: two 8-row groups, 32 bytes of dY
            tc_mma_ss(d_tmem, smem_desc_mn_sw128(a_addr + kk * 2 * kKGroup, kMnAtom, kKGroup),
                      smem_desc_sw128(b_addr + kk * 32), idesc, (j | kk) != 0);
          tc_commit(&sm->empty[st]);  // both tiles of the stage free once these MMAs have read them
        }
        if (!ok) break;
        tc_commit(&sm->acc_full[acc]);
      }
    }
  } else if (warp < kEpiWarps) {
    // ------------------------------------------------ epilogue: TMEM -> dX (or fp32 partials)
    const EpiOut o{dx, cols, m_total, part, tile_count, err};
    uint32_t ucount = 0;
    for (int u = blockIdx.x; u < wk.units; u += gridDim.x, ++ucount) {
      const int acc = ucount & 1;
      if (!wait_or_abort(&sm->acc_full[acc], (ucount >> 1) & 1, sm, err)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + acc * kAccCols;
      epilogue_unit<kTileM>(wk, u, taddr, out_stage, sm, &sm->acc_empty[acc], o, gbase);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

int dx_splits(int64_t rows, int64_t cols, int64_t m, int num_sms) {
  return reduction_splits((cols / kTileN) * ((m + kTileM - 1) / kTileM), rows / kTileR, num_sms);
}

template <bool kDQ, bool kScaleTma, int kBook>
cudaError_t launch_variant(const Scales& s, int rows, int cols, int m, int splits, const CUtensorMap& ymap,
                           const CUtensorMap& wmap, const CUtensorMap& smap, __nv_bfloat16* dx, float* part,
                           unsigned* counters, unsigned* err, int grid, cudaStream_t stream) {
  static std::atomic<uint64_t> attr_done{0};  // shared-memory opt-in, once per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!(attr_done.load() & (1ull << dev))) {
    cudaError_t e = cudaFuncSetAttribute(gemm_dx_kernel<kDQ, kScaleTma, kBook>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(1ull << dev);
  }
  const cudaError_t e = launch_pdl(gemm_dx_kernel<kDQ, kScaleTma, kBook>, dim3(grid), dim3(kThreads), kSmemBytes, stream,
                                   s, rows, cols, m, splits, ymap, wmap, smap, dx, part, counters, err);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

size_t gemm_dx_workspace_bytes(int64_t rows, int64_t cols, int64_t m) {
  const int sp = dx_splits(rows, cols, m, sm_count());
  return split_workspace_bytes((cols / kTileN) * ((m + kTileM - 1) / kTileM), sp);
}

cudaError_t launch_gemm_dx(const uint8_t* packed, const Scales& s, int64_t rows, int64_t cols, const void* dy,
                           int64_t m, void* dx, void* workspace, unsigned* err, cudaStream_t stream, int num_sms) {
  if (rows > INT32_MAX || cols > INT32_MAX || m > INT32_MAX) return cudaErrorInvalidValue;
  if (rows % kTileR != 0 || cols % kTileN != 0) return cudaErrorInvalidValue;
  const bool dq = s.absmax == nullptr;
  const int64_t rb = cols / kBlock;
  CUtensorMap ymap, wmap, smap;
  if (!make_map(&ymap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dy, rows, m, kTileR, kTileM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, packed, cols / 2, rows, 32, kTileR,
                CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorNotSupported;
  const void* sbase = dq ? (const void*)s.q : (const void*)s.absmax;
  const size_t srow = dq ? (size_t)rb : (size_t)rb * 4;
  bool scale_tma = srow % 16 == 0 && reinterpret_cast<uintptr_t>(sbase) % 16 == 0;
  if (scale_tma)
    scale_tma = dq ? make_map(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, sbase, rb, rows, 16, kTileR,
                              CU_TENSOR_MAP_SWIZZLE_NONE)
                   : make_map(&smap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, sbase, rb, rows, 4, kTileR,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!scale_tma) smap = wmap;  // unused by the kernel variant
  const int splits = dx_splits(rows, cols, m, num_sms);
  const int64_t ntiles = (cols / kTileN) * ((m + kTileM - 1) / kTileM);
  const int64_t units = ntiles * splits;
  const int grid = (int)(units < num_sms ? units : num_sms);
  unsigned* counters = nullptr;
  float* part = nullptr;
  if (splits > 1) {
    const size_t cbytes = ((size_t)ntiles * 4 + 255) & ~(size_t)255;
    counters = static_cast<unsigned*>(workspace);
    part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + cbytes);
  }
  auto* dxb = static_cast<__nv_bfloat16*>(dx);
  const int R = (int)rows, C = (int)cols, M = (int)m;
  if (dq && scale_tma)
    return s.book ? launch_variant<true, true, 1>(s, R, C, M, splits, ymap, wmap, smap, dxb, part, counters, err, grid, stream) : launch_variant<true, true, 0>(s, R, C, M, splits, ymap, wmap, smap, dxb, part, counters, err, grid, stream);
  if (dq)
    return s.book ? launch_variant<true, false, 1>(s, R, C, M, splits, ymap, wmap, smap, dxb, part, counters, err, grid, stream) : launch_variant<true, false, 0>(s, R, C, M, splits, ymap, wmap, smap, dxb, part, counters, err, grid, stream);
  if (scale_tma)
    return s.book ? launch_variant<false, true, 1>(s, R, C, M, splits, ymap, wmap, smap, dxb, part, counters, err, grid, stream) : launch_variant<false, true, 0>(s, R, C, M, splits, ymap, wmap, smap, dxb, part, counters, err, grid, stream);
  return s.book ? launch_variant<false, false, 1>(s, R, C, M, splits, ymap, wmap, smap, dxb, part, counters, err, grid, stream) : launch_variant<false, false, 0>(s, R, C, M, splits, ymap, wmap, smap, dxb, part, counters, err, grid, stream);
}

}  // namespace nf4
