// umma.cuh -- pieces shared by the tcgen05 GEMM kernels (Y = X . Wc^T and its
// input gradient dX = dY . Wc): shared-memory and instruction descriptors, MMA
// issue and commit, TMA tile loads, TMEM loads, bounded pipeline waits, the
// persistent work split, the accumulator epilogue, and host-side tensor maps.
//
// Both kernels keep one accumulator tile of 128 output columns (UMMA M, TMEM
// lanes) x 256 activation rows (UMMA N, TMEM columns; the forward takes 64 at small M) and reduce over stages of
// 64.  Both write a bf16 row-major output [m, ldy].
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "nf4_common.cuh"

namespace nf4 {
namespace umma {

constexpr int kTileN = 128;  // output columns per tile (UMMA M, TMEM lanes)
constexpr int kTileM = 256;  // activation rows per tile (UMMA N, fp32 TMEM columns); the forward GEMM also uses 64
constexpr int kAccCols = kTileM;
constexpr int kEpiWarps = 4;                  // warps 0..3 read TMEM lanes 32w..32w+31
constexpr int kStageOutBytes = 32 * 32 * 2;   // per epilogue warp: 32 rows x 32 columns of bf16
constexpr int kMaxSplits = 4;                 // reduction splits of one output tile (reduction_splits)

// ------------------------------------------------------------------ descriptors

// K-major operand, 128-byte swizzle: rows of 128 B (64 bf16 along the
// reduction), 8-row groups 1024 B apart
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fffu);          // start address
  d |= (uint64_t)1 << 16;                          // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;                // stride byte offset: next 8-row group
  d |= (uint64_t)1 << 46;                          // descriptor version (Blackwell)
  d |= (uint64_t)2 << 61;                          // layout: SWIZZLE_128B
  return d;
}

// MN-major operand, 128-byte swizzle: a swizzle atom is 8 reduction rows of
// 128 B, each row 64 consecutive bf16 along M; `mn_stride` bytes separate the
// atoms along M (leading byte offset), `k_stride` bytes the 8-row groups along
// the reduction (stride byte offset)
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t addr, uint32_t mn_stride, uint32_t k_stride) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fffu);
  d |= (uint64_t)((mn_stride >> 4) & 0x3fffu) << 16;
  d |= (uint64_t)((k_stride >> 4) & 0x3fffu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// kind::f16 instruction descriptor: bf16 A and B, fp32 D; B K-major; A K-major
// or (a_mn) MN-major
__host__ __device__ constexpr uint32_t instr_desc(int m, int n, bool a_mn = false) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(m >> 4) << 24);
}

// ------------------------------------------------------------------ tcgen05 / TMA

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D (TMEM) (+)= A (TMEM) . B (shared memory)
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}

// D (TMEM) (+)= A (shared memory) . B (shared memory)
__device__ __forceinline__ void tc_mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t acc) {
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

// 32 lanes x 32 consecutive fp32 columns (one register per column) of this warp's subpartition.
// The load and its wait are one asm statement: the registers are defined only once the wait has
// returned, so no use of them can be scheduled in between.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns from registers, then wait for the stores to land
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// ------------------------------------------------------------------ bounded pipeline waits

// every kernel's shared state carries an `abort` word: once set, every role leaves its loop
template <class Sm>
__device__ __forceinline__ bool aborted(Sm* sm) {
  return *(volatile int*)&sm->abort != 0;
}

// bounded wait; on failure mark the CTA aborted so every role leaves its loop.  A phase that has already
// completed returns at once (the abort word is read only when the thread would otherwise wait).
template <class Sm>
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Sm* sm, unsigned* err) {
  if (mbar_try_wait(bar, parity)) return true;
  if (aborted(sm)) return false;
  if (mbar_wait_bounded(bar, parity, err)) return true;
  *(volatile int*)&sm->abort = 1;
  return false;
}

// ------------------------------------------------------------------ persistent work split

// Work unit u = tile * splits + split: the split takes reduction stages
// [split * kps, (split + 1) * kps).  With splits > 1 the epilogue writes an
// fp32 partial tile to the workspace; once every split of the tile has written
// its partial (a counter per tile; the launch holds all units at once), split s
// adds the partials of 32-row chunks s, s + splits, ... in split order
// (deterministic) and writes those bf16 rows of Y.  Each split then arrives a
// second time; the last of those resets the counter, so the workspace is left
// ready for the next call.
struct Work {
  int ntiles_m, units, splits, kps;
  int tm;  // activation rows per tile
  __device__ int tile(int u) const { return u / splits; }
  __device__ int split(int u) const { return u % splits; }
  __device__ int n0(int u) const { return (tile(u) / ntiles_m) * kTileN; }  // first output column
  __device__ int m0(int u) const { return (tile(u) % ntiles_m) * tm; }      // first activation row
};

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory"); }

struct EpiOut {
  __nv_bfloat16* y;       // [m_total, ldy] row-major
  int ldy, m_total;
  float* part;            // split-K partial tiles (splits > 1)
  unsigned* tile_count;   // one arrival counter per output tile (splits > 1)
  unsigned* err;
};

// One work unit's accumulator (TMEM lanes = output columns n0 .. n0+127,
// columns = activation rows m0 .. m0+255) -> Y, run by warps 0..3.  Releases
// the accumulator through `acc_empty` as soon as it has been read.
// Shared memory the split reduction stages the other splits' partials in: 16 bytes per piece and epilogue
// thread; pieces = own 32-row chunks (ceil(TM / 32 / splits)) x 2 halves x (splits - 1) other partials x 4.
// With 2 to 4 splits that is at most 48 pieces (96 KB with 128 epilogue threads) for TM = 256 and 24 (48 KB)
// for TM = 64.
static_assert(kMaxSplits <= 4, "split staging size");
__host__ __device__ constexpr int split_stage_pieces(int tm) {
  int best = 0;
  for (int sp = 2; sp <= kMaxSplits; ++sp) {
    const int p = ((tm / 32 + sp - 1) / sp) * 2 * (sp - 1) * 4;
    best = p > best ? p : best;
  }
  return best;
}
__host__ __device__ constexpr int split_stage_bytes(int tm) { return split_stage_pieces(tm) * kEpiWarps * 32 * 16; }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// TM: activation rows of the tile (accumulator columns).  `stage_in`: split_stage_bytes(TM) of shared memory
// that is idle once the unit's MMAs have finished (the operand ring; with splits > 1 a CTA has a single unit, so
// nothing refills it)
template <int TM, class Sm>
__device__ __forceinline__ void epilogue_unit(const Work& wk, int u, uint32_t taddr, uint16_t* out_stage, Sm* sm,
                                              uint64_t* acc_empty, const EpiOut& o, uint8_t* stage_in) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nl = warp * 32 + lane;  // output column within the tile
  const int64_t n = (int64_t)wk.n0(u) + nl;
  const int m0 = wk.m0(u);
  uint16_t* st = out_stage + warp * (32 * 32);  // this warp's [32 m][32 n] bf16 tile
  // Y rows m0 + c*32 + r, columns n0 + warp*32 .. +31: the warp's 32x32 block goes
  // through shared memory so each lane stores 16 contiguous bytes of a Y row
  auto store_block = [&](int c) {
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int piece = lane + 32 * i;  // 128 pieces of 8 bf16
      const int r = piece >> 2, q = piece & 3;
      const int m = m0 + c * 32 + r;
      const uint4 v = *reinterpret_cast<const uint4*>(st + r * 32 + q * 8);
      if (m < o.m_total) *reinterpret_cast<uint4*>(o.y + (int64_t)m * o.ldy + (n - lane) + q * 8) = v;
    }
    __syncwarp();
  };
  if (wk.splits == 1) {
#pragma unroll 1
    for (int c = 0; c < TM / 32; ++c) {
      uint32_t v[32];
      tmem_ld32(taddr + c * 32, v);
#pragma unroll
      for (int j = 0; j < 32; ++j) st[j * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j])));
      store_block(c);
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acc_empty);
    return;
  }
  // Split reduction.  The fp32 partial of this unit goes to the workspace laid out [m/4][n_local][4] (each
  // 16-byte access of a warp covers 32 consecutive n, 512 contiguous bytes), except the 32-row chunks this
  // split reduces itself (c = split, split + splits, ...): those stay in TMEM until the reduction.
  const int my = wk.split(u);
  float* mine = o.part + (size_t)u * (kTileN * TM);
#pragma unroll 1
  for (int c = 0; c < TM / 32; ++c) {
    if (c % wk.splits == my) continue;
    uint32_t v[32];
    tmem_ld32(taddr + c * 32, v);
#pragma unroll
    for (int j = 0; j < 32; j += 4)
      __stcg(reinterpret_cast<float4*>(mine + ((size_t)((c * 32 + j) / 4) * kTileN + nl) * 4),
             make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]),
                         __uint_as_float(v[j + 3])));
  }
  __threadfence();
  epi_bar();
  // every split of the tile waits for all partials (the splits of a tile are co-resident: the
  // grid holds every unit at once), then finishes its share of the 32-row chunks
  unsigned second = 0;  // (thread 0) this split's second arrival, read only after the reduction
  if (threadIdx.x == 0) {
    atomicAdd(&o.tile_count[wk.tile(u)], 1u);
    const unsigned long long t0 = global_ns();
    while (*(volatile unsigned*)&o.tile_count[wk.tile(u)] < (unsigned)wk.splits) {
      if (global_ns() - t0 > kWaitLimitNs) {
        atomicOr(o.err, kErrTimeout);
        *(volatile int*)&sm->abort = 1;
        break;
      }
      __nanosleep(64);
    }
    // second arrival: the split that completes 2 * splits has seen every split pass the wait
    // above, so it can reset the counter for the next call (at the end, off the critical path)
    if (!aborted(sm)) second = atomicAdd(&o.tile_count[wk.tile(u)], 1u) + 1u;
  }
  epi_bar();
  if (!aborted(sm)) {
    __threadfence();
    const float* tp = o.part + (size_t)wk.tile(u) * wk.splits * (kTileN * TM);
    // Every other split's partial of this split's chunks, copied into shared memory with all copies in flight
    // at once (one round of L2 latency), piece p of this thread at stage_in + (p * 128 + nl) * 16.
    const uint32_t stage = smem_u32(stage_in);
    fence_proxy_async_smem();  // the ring was last written by TMA and read by the MMAs
    int pc = 0;
#pragma unroll 1
    for (int c = my; c < TM / 32; c += wk.splits)
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int q = 0; q < kMaxSplits - 1; ++q) {
          const int sp = q + (q >= my);
          if (sp < wk.splits) {
#pragma unroll
            for (int j = 0; j < 4; ++j, ++pc)
              cp_async16(stage + (uint32_t)(pc * (kEpiWarps * 32) + nl) * 16u,
                         tp + (size_t)sp * (kTileN * TM) + ((size_t)(c * 8 + h * 4 + j) * kTileN + nl) * 4);
          }
        }
    asm volatile("cp.async.commit_group;\n cp.async.wait_group 0;" ::: "memory");
    const float4* staged = reinterpret_cast<const float4*>(stage_in);
    pc = 0;
#pragma unroll 1
    for (int c = my; c < TM / 32; c += wk.splits) {
      uint32_t v[32];
      tmem_ld32(taddr + c * 32, v);  // this split's own partial of the chunk
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // 16 rows at a time
        float4 t[kMaxSplits - 1][4];
#pragma unroll
        for (int q = 0; q < kMaxSplits - 1; ++q) {
          const int sp = q + (q >= my);
          if (sp < wk.splits) {
#pragma unroll
            for (int j = 0; j < 4; ++j, ++pc) t[q][j] = staged[pc * (kEpiWarps * 32) + nl];
          }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          // partials added in split order 0, 1, ..., splits - 1
          float4 acc4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int sp = 0; sp < kMaxSplits; ++sp) {
            if (sp >= wk.splits) break;
            // split sp's partial: this split's own (TMEM) or the loads of slot sp (sp < my) / sp - 1 (sp > my);
            // every array index below is a compile-time constant
            float4 val;
            if (sp == my) {
              const int r = (h * 4 + j) * 4;
              val = make_float4(__uint_as_float(v[r]), __uint_as_float(v[r + 1]), __uint_as_float(v[r + 2]),
                                __uint_as_float(v[r + 3]));
            } else if (sp < my) {
              val = t[sp < kMaxSplits - 1 ? sp : kMaxSplits - 2][j];
            } else {
              val = t[sp > 0 ? sp - 1 : 0][j];
            }
            if (sp == 0) {
              acc4 = val;
            } else {
              acc4.x += val.x;
              acc4.y += val.y;
              acc4.z += val.z;
              acc4.w += val.w;
            }
          }
          const int r = (h * 4 + j) * 4;  // row within the chunk
          st[(r + 0) * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(acc4.x));
          st[(r + 1) * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(acc4.y));
          st[(r + 2) * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(acc4.z));
          st[(r + 3) * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(acc4.w));
        }
      }
      store_block(c);
    }
  }
  if (threadIdx.x == 0 && second == 2u * (unsigned)wk.splits) o.tile_count[wk.tile(u)] = 0;
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(acc_empty);  // TMEM no longer needed
}

// ------------------------------------------------------------------ host side

// 2-D tiled tensor map (no swizzle unless asked); false if the driver refuses it
bool make_map(CUtensorMap* map, CUtensorMapDataType type, size_t esize, const void* base, uint64_t inner,
              uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);

// Reduction splits: enough work units to cover the SMs when there are few
// output tiles; the split count divides the number of stages and leaves each
// split at least 8 stages.
int reduction_splits(int64_t ntiles, int64_t stages, int num_sms);

// bytes of the split-K workspace: one counter per tile, then the fp32 partials of tm-row tiles
size_t split_workspace_bytes(int64_t ntiles, int splits, int tm = kTileM);

int sm_count();

}  // namespace umma
}  // namespace nf4
