// gemm_sm100.cu -- prefill GEMM Y = X . Wc^T on tcgen05 tensor cores.
//
// "bitsandbytes" (ozercemkelahmet.com/tools), "How it works" Step 5: matrix
// hardware works best on 16-bit numbers, so each NF4 block is expanded back to
// 16-bit (bf16_rn(RN(code[i] * a)), compute dtype bfloat16 per "bitsandbytes
// quantization tutorial", mljourney.com) and then multiplied.  Here the
// expansion happens tile by tile in shared memory, and the multiply is a
// tcgen05 bf16 x bf16 -> fp32 MMA with the accumulator in tensor memory.
//
// Tile: 128 weight rows (UMMA M, operand A) x TM activation rows (UMMA N,
// operand B; TM = 256, or 64 while m <= 64) x 64 k per pipeline stage (one
// level-1 block per weight row).  D[n, m] lives in TMEM (lane = weight row,
// column = activation row, TM columns); the decoded weight tile goes straight
// into TMEM too (32 columns per stage of the operand ring: lane = weight row,
// column j = codes 2j, 2j+1 as bf16x2), so the MMA reads only the activation
// tile from shared memory.  The issuing thread is the pipeline's critical path
// (each tcgen05 instruction and barrier test costs it tens of cycles), so a
// stage's two tiles share one full and one empty barrier.  One persistent CTA
// per SM walks the tiles; warp roles:
//   warps 0-3   epilogue: tcgen05.ld -> bf16 -> Y (warp w reads TMEM lanes 32w..)
//   warps 4..4+4G-1  dequant producers, G groups of four taking stages in
//               turn: thread p decodes weight row p of the stage (64 codes)
//               with the byte-permute tables and stores it to its TMEM lane
//               (tcgen05.st); a decode is a long dependent chain per thread,
//               so the groups in flight are what keep the issue slots busy
//   next warp   TMA producer: activation tile (TM x 64 bf16, 128B swizzle)
//   next warp   TMEM allocator and MMA issuer (one elected thread)
//   last warp   TMA producer: packed codes and 16-byte scale chunks
// With a low-rank adapter (QLoRA: "bitsandbytes quantization tutorial",
// "QLoRA: Fine-Tuning a 4-bit Model") each output tile runs one more stage:
// the producers put [B | B] rows of the up map in the TMEM slot, the TMA warp
// loads the down map's [hi | lo] rows (lora_down.cu) in place of an activation
// tile, and the MMA reduces over 2r, so the adapter lands in the same
// accumulator.  The descriptors, MMA wrappers, work split and epilogue shared
// with the input-gradient kernel live in umma.cuh.
// Every mbarrier wait is bounded; on timeout the device error word is set and
// the roles leave their loops, so a fault cannot hang the GPU.
#include <cuda.h>

#include <atomic>

#include "nf4_common.cuh"
#include "nf4_decode.cuh"
#include "internal.h"
#include "umma.cuh"

namespace nf4 {
namespace {

using namespace umma;

constexpr int kTileK = 64;        // k per stage (128 bytes of bf16: one swizzle atom)
// producer groups of four warps, one stage each in turn (3 or 4 groups -- more warps with fewer registers each --
// measured 3 to 25 % slower at every shape)
constexpr int kGroups = 2;
constexpr int kWStages = 6;  // packed-code + scale ring (TMA from HBM), deeper to hide its latency
constexpr int kWBytes = kTileN * kTileK / 2;  // 4 KB: packed codes of the weight tile
constexpr int kSBytes = kTileN * 16;          // 2 KB: 16-byte scale chunk per weight row
constexpr int kProdWarp0 = 4;                 // producers: warps 4 .. 4 + 4 kGroups - 1
constexpr int kTmaWarp = kProdWarp0 + 4 * kGroups;  // activation tiles
constexpr int kMmaWarp = kTmaWarp + 1;
constexpr int kTmaWWarp = kTmaWarp + 2;             // packed codes and scales
constexpr int kThreads = (kTmaWWarp + 1) * 32;
constexpr int kStagesMax = 8;

// Per activation-tile width TM (the UMMA N: 256, or 64 for up to 64 activation rows, where a 256-wide tile would
// spend three quarters of every MMA on padding rows): the operand ring and the TMEM budget.  Stage s of the ring
// is an activation tile in shared memory (TMA) and a decoded weight tile in TMEM columns (producer warps) that
// fill and empty together: one full barrier (the TMA's bytes + the four producer warps of the stage's group) and
// one empty barrier (one tcgen05.commit), so the single MMA-issuing thread waits once and commits once per stage.
template <int TM>
struct TileCfg {
  static constexpr int kStages = TM == 256 ? 5 : 8;  // operand ring depth
  static constexpr int kBBytes = TM * kTileK * 2;    // activation tile (operand B): 32 KB at TM = 256
  static constexpr int kRingBytes = kStages * kBBytes + kWStages * (kWBytes + kSBytes);  // A lives in TMEM
  static constexpr int kTmemCols = TM + kStages * 32 <= 256 ? 256 : 512;  // accumulator + A ring, a power of 2
  static constexpr size_t kSmemBytes = (size_t)kRingBytes + kEpiWarps * kStageOutBytes + 1024 /*align*/ +
                                       2048 /*barriers, lut*/;
  static_assert(kStages * kBBytes >= split_stage_bytes(TM), "split reduction staging fits in the operand ring");
  static_assert(TM + kStages * 32 <= kTmemCols, "TMEM: accumulator + A ring");
  static_assert(kStages <= kStagesMax, "barrier array");
};

struct Smem {  // placed after the 1024-aligned stage buffers
  uint64_t wfull[kWStages];   // packed codes + scale chunk landed (TMA)
  uint64_t wempty[kWStages];  // codes read by the producer warps
  uint64_t full[kStagesMax];   // activation tile landed (TMA) and decoded weight tile written (producer warps)
  uint64_t empty[kStagesMax];  // both consumed by the stage's MMAs (tcgen05.commit)
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
  int abort;
  float unit_lut[256];
};

// ------------------------------------------------------------------ kernel

#ifdef NF4_TRACE  // diagnostics build only: per-CTA wall-clock stamps of pipeline milestones
__device__ unsigned long long g_trace[1024 * 16];
#define NF4_STAMP(slot) (g_trace[blockIdx.x * 16 + (slot)] = global_ns())
#else
#define NF4_STAMP(slot) ((void)0)
#endif

template <bool kDQ, bool kScaleTma, int kBook, int TM>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(Scales s, int rows, int cols, int m_total, int splits, const __grid_constant__ CUtensorMap xmap,
                const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                __nv_bfloat16* __restrict__ y, float* __restrict__ part, unsigned* __restrict__ tile_count,
                unsigned* err, const __grid_constant__ CUtensorMap tmap, const __nv_bfloat16* __restrict__ lora_up,
                int lora_r) {
  using Cfg = TileCfg<TM>;
  constexpr int kStages = Cfg::kStages, kBBytes = Cfg::kBBytes, kRingBytes = Cfg::kRingBytes;
  constexpr int kTmemCols = Cfg::kTmemCols;
  constexpr int kAccColsT = TM;  // accumulator columns; the A ring follows
  extern __shared__ uint8_t smem_raw[];
  pdl_launch_dependents();
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;  // 1024-aligned stage buffers (swizzle atoms)
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t b_smem0 = base;
  const uint32_t w_smem0 = b_smem0 + kStages * kBBytes, s_smem0 = w_smem0 + kWStages * kWBytes;
  const uint8_t* w_gen0 = gbase + (w_smem0 - base);
  const uint8_t* s_gen0 = gbase + (s_smem0 - base);
  uint16_t* out_stage = reinterpret_cast<uint16_t*>(gbase + kRingBytes);  // epilogue transpose
  Smem* sm = reinterpret_cast<Smem*>(gbase + kRingBytes + kEpiWarps * kStageOutBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Work wk;
  wk.ntiles_m = (m_total + TM - 1) / TM;
  wk.tm = TM;
  wk.splits = splits;
  wk.units = (rows / kTileN) * wk.ntiles_m * splits;
  wk.kps = cols / kTileK / splits;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kWStages; ++i) {
      mbar_init(&sm->wfull[i], 1);   // TMA arrive.expect_tx
      mbar_init(&sm->wempty[i], 4);  // the 4 producer warps of the stage's group
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
  // Everything above is on-chip set-up; from here on global memory is read and written.  With an adapter
  // (lora_r > 0) the launch before this one is the down map, which let this grid start only after its own
  // predecessor had finished: X, the weight and the outputs are safe to touch now, and only the adapter
  // stage's load of the down map's output waits for that grid (in the activation TMA warp).
  if (lora_r == 0) pdl_wait();
  const uint32_t tmem = sm->tmem_base;
  if (threadIdx.x == 0) NF4_STAMP(0);

  if (warp >= kProdWarp0 && warp < kTmaWarp) {
    // ------------------------------------------------ dequant producers
    const int group = (warp - kProdWarp0) >> 2;          // 0 .. kGroups - 1: stages in turn
    const int p = ((warp - kProdWarp0) & 3) * 32 + lane;  // weight row within the tile
    const float mu = kDQ ? *s.mean : 0.0f;
    const int64_t rb = cols / kBlock;
    const DecodeMul dm = decode_mul();
    uint32_t it = 0, wit = 0;  // stages (A ring, group alternation); weight stages (code ring)
    for (int u = blockIdx.x; u < wk.units; u += gridDim.x) {
      const int64_t row = (int64_t)wk.n0(u) + p;
      const int ks0 = wk.split(u) * wk.kps;
      const int ks1 = ks0 + wk.kps + (lora_r > 0 && wk.split(u) == 0 ? 1 : 0);  // + the adapter stage
      for (int ks = ks0; ks < ks1; ++ks, ++it) {
        const bool adapter = ks == ks0 + wk.kps;
        if (!adapter) ++wit;
        if ((int)(it % kGroups) != group) continue;
        const int as = it % kStages;
        const uint32_t aph = (it / kStages) & 1;
        if (adapter) {
          // adapter stage: this row of the up map B[n, 0..r) twice, [B | B] in the first r columns of the A slot
          // (zeros after), against [T_hi | T_lo] of the down map
          uint32_t r[32];
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            uint4 v = make_uint4(0, 0, 0, 0);
            const int e = 2 * j;  // first element of these 8
            if (e < 2 * lora_r)
              v = __ldg(reinterpret_cast<const uint4*>(lora_up + row * lora_r + (e < lora_r ? e : e - lora_r)));
            r[j] = v.x;
            r[j + 1] = v.y;
            r[j + 2] = v.z;
            r[j + 3] = v.w;
          }
          if (!wait_or_abort(&sm->empty[as], aph ^ 1, sm, err)) break;
          const uint32_t ta = tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(kAccColsT + as * 32);
          tmem_st32(ta, r);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm->full[as]);
          continue;
        }
        const int ws = (wit - 1) % kWStages;
        const uint32_t wph = ((wit - 1) / kWStages) & 1;
        if (!wait_or_abort(&sm->wfull[ws], wph, sm, err)) break;  // codes + scale chunk landed
        const uint4* wsrc = reinterpret_cast<const uint4*>(w_gen0 + ws * kWBytes + p * 32);
        const uint4 w0 = wsrc[0], w1 = wsrc[1];
        const uint8_t* sc = s_gen0 + ws * kSBytes + p * 16;
        const int64_t b = row * rb + ks;  // level-1 block of this row and stage
        const uint32_t qcode = kDQ && kScaleTma ? sc[ks & 15] : 0u;
        const float plain = !kDQ && kScaleTma ? reinterpret_cast<const float*>(sc)[ks & 3] : 0.0f;
        // the slot is refilled by TMA (async proxy) after these generic-proxy reads: order them first
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->wempty[ws]);  // the code slot may be refilled
        float a;
        if (kDQ)
          a = dq_absmax(sm->unit_lut[kScaleTma ? qcode : s.q[b]], __ldg(s.scale + b / kDqBlock), mu);
        else
          a = kScaleTma ? plain : __ldg(s.absmax + b);
        const Table T = make_table<kBook>(a);
        const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        uint32_t r[32];  // column j of the row: codes 2j, 2j+1 as bf16x2
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t d[4];
          decode_word(words[c], T, d, dm);
          r[4 * c] = d[0];
          r[4 * c + 1] = d[1];
          r[4 * c + 2] = d[2];
          r[4 * c + 3] = d[3];
        }
        if (!wait_or_abort(&sm->empty[as], aph ^ 1, sm, err)) break;  // the MMAs left this slot
        tmem_st32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(kAccColsT + as * 32), r);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->full[as]);
      }
      if (aborted(sm)) break;
    }
  } else if (warp == kTmaWarp) {
    // ------------------------------------------------ TMA: activation tiles
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap)) : "memory");
      uint32_t it = 0;
      for (int u = blockIdx.x; u < wk.units && !aborted(sm); u += gridDim.x) {
        const int ks0 = wk.split(u) * wk.kps;
        const int ks1 = ks0 + wk.kps + (lora_r > 0 && wk.split(u) == 0 ? 1 : 0);
        const int m0 = wk.m0(u);
        for (int ks = ks0; ks < ks1; ++ks, ++it) {
          const int xs = it % kStages;
          if (!wait_or_abort(&sm->empty[xs], ((it / kStages) & 1) ^ 1, sm, err)) break;
          if (it == 0) NF4_STAMP(1);
          mbar_expect_tx(&sm->full[xs], kBBytes);
          if (ks == ks0 + wk.kps) {  // adapter stage: the down map's [hi | lo | 0] rows, 64 wide
            pdl_wait();              // the down-map grid has finished and its writes are visible
            tma_load_2d(b_smem0 + xs * kBBytes, &tmap, 0, m0, &sm->full[xs]);
          } else {
            tma_load_2d(b_smem0 + xs * kBBytes, &xmap, ks * kTileK, m0, &sm->full[xs]);
          }
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
        const int n0 = wk.n0(u);
        for (int ks = ks0; ks < ks0 + wk.kps; ++ks, ++it) {
          const int ws = it % kWStages;
          if (!wait_or_abort(&sm->wempty[ws], ((it / kWStages) & 1) ^ 1, sm, err)) break;
          mbar_expect_tx(&sm->wfull[ws], kWBytes + (kScaleTma ? kSBytes : 0));
          tma_load_2d(w_smem0 + ws * kWBytes, &wmap, ks * (kTileK / 2), n0, &sm->wfull[ws]);
          // the 16-byte scale chunk holding this stage's block: 16 codes or 4 fp32
          if (kScaleTma)
            tma_load_2d(s_smem0 + ws * kSBytes, &smap, kDQ ? (ks & ~15) : (ks & ~3), n0, &sm->wfull[ws]);
        }
      }
      const uint32_t issued = it;  // drain the copies still in flight
      for (uint32_t j = (issued > kWStages ? issued - kWStages : 0); j < issued; ++j)
        mbar_wait_bounded(&sm->wfull[j % kWStages], (j / kWStages) & 1, err);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc(kTileN, TM);
      uint32_t it = 0, ucount = 0;
      for (int u = blockIdx.x; u < wk.units && !aborted(sm); u += gridDim.x, ++ucount) {
        const int acc = 0;  // one accumulator: the A ring takes the other TMEM columns
        if (!wait_or_abort(&sm->acc_empty[acc], (ucount & 1) ^ 1, sm, err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * kAccColsT;
        bool ok = true;
        const int nst = wk.kps + (lora_r > 0 && wk.split(u) == 0 ? 1 : 0);  // + the adapter stage
        for (int j = 0; j < nst; ++j, ++it) {
          const int st = it % kStages;
          if (!wait_or_abort(&sm->full[st], (it / kStages) & 1, sm, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (it == 0) NF4_STAMP(2);
          const uint32_t a_tm = tmem + (uint32_t)(kAccColsT + st * 32), b_addr = b_smem0 + st * kBBytes;
          const int nkk = j < wk.kps ? kTileK / 16 : lora_r / 8;  // the adapter stage reduces over 2r only
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk)  // 16 bf16 per MMA along k: 8 TMEM columns, 32 smem bytes
            if (kk < nkk) tc_mma_ts(d_tmem, a_tm + kk * 8, smem_desc_sw128(b_addr + kk * 32), idesc, (j | kk) != 0);
          tc_commit(&sm->empty[st]);  // both tiles of the stage free once these MMAs have read them
        }
        if (!ok) break;
        NF4_STAMP(3);
        tc_commit(&sm->acc_full[acc]);  // accumulator ready for the epilogue
      }
    }
  } else if (warp < kEpiWarps) {
    // ------------------------------------------------ epilogue: TMEM -> Y (or fp32 partials)
    const EpiOut o{y, rows, m_total, part, tile_count, err};
    uint32_t ucount = 0;
    for (int u = blockIdx.x; u < wk.units; u += gridDim.x, ++ucount) {
      const int acc = 0;
      if (!wait_or_abort(&sm->acc_full[acc], ucount & 1, sm, err)) break;
      tc_fence_after();
      if (threadIdx.x == 0) NF4_STAMP(4);
      const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + acc * kAccColsT;
      epilogue_unit<TM>(wk, u, taddr, out_stage, sm, &sm->acc_empty[acc], o, gbase);
      if (threadIdx.x == 0) NF4_STAMP(6);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) NF4_STAMP(7);
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

// up to this many activation rows nf4_gemm runs the GEMV kernel (one mma.sync n-tile; two n-tiles for 9-16 rows
// measured 43.3 us against the 64-row tcgen05 tile's 37.5 us at 14336x4096, m = 16)
constexpr int64_t kGemvMaxRows = 8;

// activation rows per tile: 64 while they cover m (the MMA's N then carries no padding rows beyond 64), else 256
int gemm_tile_m(int64_t m) { return m <= 64 ? 64 : 256; }

int64_t gemm_tiles(int64_t rows, int64_t m) {
  const int tm = gemm_tile_m(m);
  return (rows / kTileN) * ((m + tm - 1) / tm);
}

int gemm_splits(int64_t rows, int64_t cols, int64_t m, int num_sms) {
  if (m <= kGemvMaxRows) return 1;  // served by the GEMV
  return reduction_splits(gemm_tiles(rows, m), cols / kTileK, num_sms);
}

}  // namespace

namespace umma {

bool make_map(CUtensorMap* map, CUtensorMapDataType type, size_t esize, const void* base, uint64_t inner,
              uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  EncodeTiled encode = get_encoder();
  if (encode == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  const cuuint64_t strides[1] = {(cuuint64_t)(inner * esize)};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return encode(map, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int reduction_splits(int64_t ntiles, int64_t stages, int num_sms) {
  int best = 1;
  for (int sp = 2; sp <= kMaxSplits; ++sp)
    if (stages % sp == 0 && stages / sp >= 8 && ntiles * sp <= num_sms) best = sp;
  return best;
}

size_t split_workspace_bytes(int64_t ntiles, int splits, int tm) {
  if (splits == 1) return 0;
  const size_t counters = ((size_t)ntiles * 4 + 255) & ~(size_t)255;
  return counters + (size_t)ntiles * splits * kTileN * tm * sizeof(float);
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

}  // namespace umma

size_t gemm_workspace_bytes(int64_t rows, int64_t cols, int64_t m) {
  const int sp = gemm_splits(rows, cols, m, sm_count());
  return split_workspace_bytes(gemm_tiles(rows, m), sp, gemm_tile_m(m));
}

namespace {

template <bool kDQ, bool kScaleTma, int kBook, int TM>
cudaError_t launch_variant(const Scales& s, int rows, int cols, int m, int splits, const CUtensorMap& xmap,
                           const CUtensorMap& wmap, const CUtensorMap& smap, __nv_bfloat16* y, float* part,
                           unsigned* counters, unsigned* err, int grid, cudaStream_t stream, const CUtensorMap& tmap,
                           const __nv_bfloat16* lora_up, int lora_r) {
  constexpr size_t smem = TileCfg<TM>::kSmemBytes;
  // the shared-memory opt-in is a per-device function attribute: set it once
  // per device (outside any stream capture that later calls may be part of)
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!(attr_done.load() & (1ull << dev))) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<kDQ, kScaleTma, kBook, TM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(1ull << dev);
  }
  const cudaError_t e = launch_pdl(gemm_kernel<kDQ, kScaleTma, kBook, TM>, dim3(grid), dim3(kThreads), smem, stream, s,
                                   rows, cols, m, splits, xmap, wmap, smap, y, part, counters, err, tmap, lora_up,
                                   lora_r);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int TM>
cudaError_t launch_book_scales(bool dq, bool scale_tma, int book, const Scales& s, int R, int C, int M, int splits,
                               const CUtensorMap& xmap, const CUtensorMap& wmap, const CUtensorMap& smap,
                               __nv_bfloat16* yb, float* part, unsigned* counters, unsigned* err, int grid,
                               cudaStream_t stream, const CUtensorMap& tmap, const __nv_bfloat16* up, int lora_r) {
#define NF4_GEMM_VARIANT(DQ, ST, BK)                                                                                 \
  launch_variant<DQ, ST, BK, TM>(s, R, C, M, splits, xmap, wmap, smap, yb, part, counters, err, grid, stream, tmap, \
                                 up, lora_r)
  if (dq && scale_tma) return book ? NF4_GEMM_VARIANT(true, true, 1) : NF4_GEMM_VARIANT(true, true, 0);
  if (dq) return book ? NF4_GEMM_VARIANT(true, false, 1) : NF4_GEMM_VARIANT(true, false, 0);
  if (scale_tma) return book ? NF4_GEMM_VARIANT(false, true, 1) : NF4_GEMM_VARIANT(false, true, 0);
  return book ? NF4_GEMM_VARIANT(false, false, 1) : NF4_GEMM_VARIANT(false, false, 0);
#undef NF4_GEMM_VARIANT
}

}  // namespace

namespace {

// the tcgen05 kernel for m activation rows; with lora_r > 0 each output tile adds one adapter stage
// (T = the [m, 64] bf16 down-map output [hi | lo | 0] at `t`, lora_up = B [rows, r])
cudaError_t launch_tc(const uint8_t* packed, const Scales& s, int64_t rows, int64_t cols, const void* x, int64_t m,
                      void* y, int splits, void* workspace, unsigned* err, cudaStream_t stream, int num_sms,
                      const void* t, const void* lora_up, int lora_r) {
  auto* yb = static_cast<__nv_bfloat16*>(y);
  if (rows > INT32_MAX || cols > INT32_MAX || m > INT32_MAX) return cudaErrorInvalidValue;
  const bool dq = s.absmax == nullptr;
  const int64_t rb = cols / kBlock;  // level-1 blocks per weight row
  const int tm = gemm_tile_m(m);
  CUtensorMap xmap, wmap, smap, tmap;
  if (!make_map(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, cols, m, kTileK, tm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, packed, cols / 2, rows, kTileK / 2, kTileN,
                CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorNotSupported;
  if (lora_r > 0) {
    if (!make_map(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, t, kTileK, m, kTileK, tm, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorNotSupported;
  } else {
    tmap = xmap;  // unused
  }
  // scale chunks through TMA when each row of scales is a whole number of 16-byte units
  const void* sbase = dq ? (const void*)s.q : (const void*)s.absmax;
  const size_t srow = dq ? (size_t)rb : (size_t)rb * 4;
  bool scale_tma = srow % 16 == 0 && reinterpret_cast<uintptr_t>(sbase) % 16 == 0;
  if (scale_tma)
    scale_tma = dq ? make_map(&smap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, sbase, rb, rows, 16, kTileN,
                              CU_TENSOR_MAP_SWIZZLE_NONE)
                   : make_map(&smap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, sbase, rb, rows, 4, kTileN,
                              CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!scale_tma) smap = wmap;  // unused by the kernel variant
  const int64_t ntiles = gemm_tiles(rows, m);
  const int64_t units = ntiles * splits;
  const int grid = (int)(units < num_sms ? units : num_sms);
  unsigned* counters = nullptr;
  float* part = nullptr;
  if (splits > 1) {
    const size_t cbytes = ((size_t)ntiles * 4 + 255) & ~(size_t)255;
    counters = static_cast<unsigned*>(workspace);
    part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + cbytes);
  }
  const int R = (int)rows, C = (int)cols, M = (int)m;
  const auto* up = static_cast<const __nv_bfloat16*>(lora_up);
  return tm == 64 ? launch_book_scales<64>(dq, scale_tma, s.book, s, R, C, M, splits, xmap, wmap, smap, yb, part,
                                           counters, err, grid, stream, tmap, up, lora_r)
                  : launch_book_scales<256>(dq, scale_tma, s.book, s, R, C, M, splits, xmap, wmap, smap, yb, part,
                                            counters, err, grid, stream, tmap, up, lora_r);
}

// the adapter path: its own split choice (no GEMV route for small m), the [m, 64] bf16 down-map output first
// in the workspace, the split-K scratch after it
int lora_splits(int64_t rows, int64_t cols, int64_t m, int num_sms) {
  return reduction_splits(gemm_tiles(rows, m), cols / kTileK, num_sms);
}

size_t lora_t_bytes(int64_t m) { return ((size_t)m * kTileK * 2 + 255) & ~(size_t)255; }

}  // namespace

cudaError_t launch_gemm(const uint8_t* packed, const Scales& s, int64_t rows, int64_t cols, const void* x, int64_t m,
                        void* y, void* workspace, unsigned* err, cudaStream_t stream, int num_sms) {
  // up to 8 activation rows: the decode GEMV; above, the tensor-core kernel (64-row activation tiles up to 64
  // rows, 256 above)
  if (m <= kGemvMaxRows) return launch_gemv(packed, s, rows, cols, x, (int)m, y, err, stream, num_sms);
  return launch_tc(packed, s, rows, cols, x, m, y, gemm_splits(rows, cols, m, num_sms), workspace, err, stream,
                   num_sms, nullptr, nullptr, 0);
}

size_t gemm_lora_workspace_bytes(int64_t rows, int64_t cols, int64_t m) {
  return lora_t_bytes(m) + split_workspace_bytes(gemm_tiles(rows, m), lora_splits(rows, cols, m, sm_count()),
                                                 gemm_tile_m(m));
}

cudaError_t launch_gemm_lora(const uint8_t* packed, const Scales& s, int64_t rows, int64_t cols, const void* x,
                             int64_t m, const void* lora_down, const void* lora_up, int lora_r, float lora_scale,
                             void* y, void* workspace, unsigned* err, cudaStream_t stream, int num_sms) {
  if (rows > INT32_MAX || cols > INT32_MAX || m > INT32_MAX) return cudaErrorInvalidValue;
  void* t = workspace;
  cudaError_t e = launch_lora_down(x, lora_down, m, cols, lora_r, lora_scale, t, stream);
  if (e != cudaSuccess) return e;
  void* split_ws = static_cast<uint8_t*>(workspace) + lora_t_bytes(m);
  return launch_tc(packed, s, rows, cols, x, m, y, lora_splits(rows, cols, m, num_sms), split_ws, err, stream,
                   num_sms, t, lora_up, lora_r);
}

}  // namespace nf4

#ifdef NF4_TRACE
extern "C" __attribute__((visibility("default"))) int nf4_trace_read(unsigned long long* host) {
  return (int)cudaMemcpyFromSymbol(host, nf4::g_trace, sizeof(nf4::g_trace));
}
#endif
