// gemv_stream.cu -- decode GEMV (batch 1..8) over one or many NF4 weights in one persistent launch.
//
// "bitsandbytes" (ozercemkelahmet.com/tools), "How it works" Step 5: each block
// is expanded back to 16-bit with its scale and the code book, then
// multiplied; compute dtype bfloat16 ("bitsandbytes quantization tutorial",
// mljourney.com, "4-bit Loading with NF4").  Effective weight
// Wc = bf16_rn(RN(code[idx] * a)), y[b, n] = bf16_rn(sum_k Wc[n, k] x[b, k]),
// fp32 accumulation.
//
// Work: one launch takes a list of items (weight, input x, output y), all with the same 4-bit code book (NF4, or
// FP4 -- the kernel is templated on the 16 levels).  The
// items' 16-row tiles form one sequence; the host cuts it into one contiguous
// range per CTA (one CTA per SM) with equal work to within one tile, so a
// whole-model pass over hundreds of weights is a single launch.
//
// Inside a CTA every tile is cut into groups of four warp steps (a warp step is
// 16 rows x 256 columns); the CTA's groups, counted across its tiles, go round
// robin to its 16 warps, so all warps stay busy through tile boundaries.  In a
// step, lane (g = lane/4, t = lane%4) owns rows g and g + 8 and level-1 block t
// of the step: 32 code bytes per row, two 16-byte loads each.  Loads run one
// step ahead in registers, and upcoming tiles are prefetched into L2 with bulk
// prefetches (one instruction per tile, no registers or shared memory held),
// so the register loads meet L2 instead of HBM.
//
// Decode (the limiter at batch 1): the 16-bit weight bf16_rn(code * a) comes
// from two paths on different pipes, mixed per word of 8 codes:
//   - byte-permute pools (ALU): the block's 16 bf16 values are built once and
//     a packed word is decoded with byte permutes (nf4_decode.cuh);
//   - a shared table of fp32 code pairs indexed by the code byte (one copy per
//     lane: no bank conflicts): one shared load, one paired multiply by a and
//     one bf16x2 convert give two weights.
// The decoded pairs are the A operand of mma.sync m16n8k16 (weights on M,
// batch <= 8 on N).  Every lane loads an activation row (lanes past the batch repeat its last row), so the
// loads need no predicate; the extra output columns are never read.
//
// Partial sums: a warp accumulates its groups of a tile, then leaves its fp32
// partial in one of four shared slots (by tile); the warp that completes a
// tile's count adds the partials in group order -- the same order whichever
// CTA or warp holds the groups, so results are deterministic and identical to
// a single-weight launch -- and writes y.
#include <algorithm>

#include "nf4_common.cuh"
#include "nf4_decode.cuh"
#include "internal.h"

namespace nf4 {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kStepCols = 256;                 // columns per warp step (4 level-1 blocks)
constexpr int kGroupSteps = 4;                 // steps per round-robin group
constexpr int kSlots = 4;                      // partial-sum slots (tiles in flight per CTA)
constexpr int kPairTableBytes = 256 * 32 * 8;  // fp32 code pairs, one copy per lane
constexpr int kSlotFloats = kWarps * 16 * 8;   // one slot: [group in tile][row][batch column]
constexpr int kMaxCtas = 160;
constexpr int kRestBytes = (kSlots * kSlotFloats + 512) * 4;  // partial slots + dq unit table
constexpr int kSmemBytes = 65536 + kPairTableBytes + kRestBytes;  // table + its alignment slack + the rest

constexpr int kPlain = 0;  // item kinds: fp32 absmax / double quant E4M3 / double quant int8
constexpr int kDqE4M3 = 1;
constexpr int kDqInt8 = 2;

struct Item {
  const uint8_t* packed;
  const void* scl;      // fp32 absmax (plain) or 8-bit codes (double quant)
  const float* scale2;  // second-level block absmax (double quant)
  const float* mean;    // device pointer to the removed mean (double quant)
  const __nv_bfloat16* x;
  __nv_bfloat16* y;
  int32_t cols;  // K
  int32_t kind;
};

template <int kMax>
struct Params {
  Item item[kMax];
  int32_t tile_end[kMax];        // cumulative 16-row tile counts
  int32_t cta_tile[kMaxCtas + 1];  // CTA c takes tiles [cta_tile[c], cta_tile[c + 1])
  int32_t count;
  int32_t batch;
};

__constant__ float c_code_stream[2][16] = {NF4_CODE_INIT, FP4_CODE_INIT};  // by code book: NF4, FP4

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two weights through the pair table: the fp32 pair (code[hi nibble], code[lo nibble]) at shared address `addr`,
// each multiplied by a (RN), converted to bf16x2 (first element in the low half).  Two scalar multiplies: the
// paired f32x2 multiply measured at half the rate when interleaved with mma.sync.
__device__ __forceinline__ uint32_t table_pair(uint32_t addr, float a) {
  float c0, c1;
  asm("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(c0), "=f"(c1) : "r"(addr));
  return pack_bf16x2(__fmul_rn(c0, a), __fmul_rn(c1, a));
}

// 8 codes of one packed word through the pair table: out[b] = (e_2b, e_2b+1).  The table is 64 KB aligned in
// shared memory, so one byte permute forms the whole address: byte 0 = 8 * lane, byte 1 = the code byte, bytes 2-3
// = the table's base (all carried in `lane_base`).
__device__ __forceinline__ void table_decode(uint32_t w, float a, uint32_t lane_base, uint32_t (&out)[4]) {
#pragma unroll
  for (int b = 0; b < 4; ++b) out[b] = table_pair(prmt(w, lane_base, 0x7604u | (b << 4)), a);
}

template <int kMax>
__device__ __forceinline__ int tile_begin(const Params<kMax>& p, int i) {
  return i > 0 ? p.tile_end[i - 1] : 0;
}

template <int kG = kGroupSteps>
__host__ __device__ __forceinline__ int tile_groups(int cols) {
  return ((cols + kStepCols - 1) / kStepCols + kG - 1) / kG;
}

// One warp's walk over its steps: groups G = warp, warp + 16, ... of the CTA (counted across its tiles), each of
// up to kGroupSteps steps of one tile.
struct Walk {
  int j;       // global tile index
  int item;    // its item
  int gbase;   // CTA-local index of tile j's first group
  int ng;      // groups of tile j
  int nsteps;  // steps of tile j
  int G;       // current group
  int s;       // current step of tile j
  int send;    // end step of the current group
  // tile j for this lane
  const uint8_t* pk;       // codes of row g, block t of step 0
  const uint8_t* sk;       // scale (4-byte) or scale code (1-byte) of row g, block t of step 0
  const __nv_bfloat16* xk; // x of activation row min(g, batch - 1) at block t of step 0
  int64_t b0;              // level-1 block index of row g, block t of step 0
  uint32_t rstride;        // code bytes between rows g and g + 8
  uint32_t sstride;        // scale bytes between rows g and g + 8
  int nbr;                 // level-1 blocks per row
};

template <int kG, int kMax>
__device__ __forceinline__ void walk_tile(const Params<kMax>& p, Walk& w, int g, int t, int batch) {
  const Item& it = p.item[w.item];
  const int64_t row = (int64_t)(w.j - tile_begin(p, w.item)) * 16 + g;
  const int esz = it.kind == kPlain ? 4 : 1;
  w.nbr = it.cols / kBlock;
  w.nsteps = (it.cols + kStepCols - 1) / kStepCols;
  w.ng = (w.nsteps + kG - 1) / kG;
  w.pk = it.packed + row * (it.cols / 2) + t * 32;
  w.b0 = row * w.nbr + t;
  w.sk = static_cast<const uint8_t*>(it.scl) + w.b0 * esz;
  w.xk = it.x + (int64_t)min(g, batch - 1) * it.cols + t * kBlock;
  w.rstride = (uint32_t)(8 * (it.cols / 2));
  w.sstride = (uint32_t)(8 * w.nbr * esz);
}

// move to group w.G (at or after the current tile); false past the CTA's range
template <int kG, int kMax>
__device__ __forceinline__ bool walk_locate(const Params<kMax>& p, Walk& w, int t_end, int g, int t, int batch) {
  bool moved = false;
  while (w.j < t_end && w.G >= w.gbase + w.ng) {
    w.gbase += w.ng;
    ++w.j;
    if (w.j >= t_end) break;
    while (w.j >= p.tile_end[w.item]) ++w.item;
    w.ng = tile_groups<kG>(p.item[w.item].cols);
    moved = true;
  }
  if (w.j >= t_end) return false;
  if (moved) walk_tile<kG>(p, w, g, t, batch);
  w.s = (w.G - w.gbase) * kG;
  w.send = min(w.s + kG, w.nsteps);
  return true;
}

struct Step {       // one warp step of one lane
  uint4 w0[2];      // 32 code bytes of row g
  uint4 w1[2];      // 32 code bytes of row g + 8
  float s0, s1;     // plain absmax, or second-level block absmax (double quant)
  uint32_t q;       // 8-bit scale codes of rows g (bits 0-7) and g + 8 (bits 8-15) (double quant)
  float mu;         // removed mean (double quant)
  float a0, a1;     // reconstructed scales of rows g and g + 8 (filled one step ahead of use)
  const __nv_bfloat16* xp;  // x at this step's block (activation row min(g, batch - 1))
  int lj;           // CTA-local tile index (-1: no step)
  int info;         // bits 0-3: the group's index in its tile modulo 16; bits 4-5: kind
};

template <int kMax>
__device__ __forceinline__ void load_step(const Params<kMax>& p, Step& d, const Walk& w, bool live, int t_begin) {
  if (!live) {
    d.lj = -1;
    return;
  }
  const Item& it = p.item[w.item];
  d.lj = w.j - t_begin;
  d.info = ((w.G - w.gbase) & 15) | (it.kind << 4);
  const int kind = it.kind;
  if (w.s * 4 + (int)(threadIdx.x & 3) >= w.nbr) {
    // ragged last step: zero codes and scale; x points at its row start (finite values, multiplied by zero)
    d.w0[0] = d.w0[1] = d.w1[0] = d.w1[1] = make_uint4(0x77777777u, 0x77777777u, 0x77777777u, 0x77777777u);
    d.s0 = d.s1 = 0.0f;
    d.q = 0;
    d.mu = 0.0f;
    d.xp = w.xk - (threadIdx.x & 3) * kBlock;
    return;
  }
  d.xp = w.xk + w.s * kStepCols;
  const uint8_t* c = w.pk + w.s * 128;
  d.w0[0] = __ldcs(reinterpret_cast<const uint4*>(c));
  d.w0[1] = __ldcs(reinterpret_cast<const uint4*>(c) + 1);
  d.w1[0] = __ldcs(reinterpret_cast<const uint4*>(c + w.rstride));
  d.w1[1] = __ldcs(reinterpret_cast<const uint4*>(c + w.rstride) + 1);
  if (kind == kPlain) {
    const float* sc = reinterpret_cast<const float*>(w.sk) + w.s * 4;
    d.s0 = __ldcs(sc);
    d.s1 = __ldcs(reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(sc) + w.sstride));
    d.q = 0;
    d.mu = 0.0f;
  } else {
    const uint8_t* sc = w.sk + w.s * 4;
    d.q = (uint32_t)__ldcs(sc) | ((uint32_t)__ldcs(sc + w.sstride) << 8);
    const int64_t b0 = w.b0 + w.s * 4;
    d.s0 = __ldg(it.scale2 + (b0 >> 8));
    d.s1 = __ldg(it.scale2 + ((b0 + 8 * w.nbr) >> 8));
    d.mu = __ldg(it.mean);
  }
}

// Bulk-prefetch tile j into L2: its codes (one contiguous range: the tile's 16 rows are consecutive) and the
// 16-byte-aligned interior of its level-1 scales or scale codes (also contiguous).
__device__ __forceinline__ void prefetch_range(const void* begin, const void* end) {
  uintptr_t a = (reinterpret_cast<uintptr_t>(begin) + 15) & ~(uintptr_t)15;
  const uintptr_t b = reinterpret_cast<uintptr_t>(end) & ~(uintptr_t)15;
  for (; a < b; a += 65536) {
    const uint32_t n = (uint32_t)(b - a < 65536 ? b - a : 65536);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"(n) : "memory");
  }
}

template <int kMax>
__device__ __forceinline__ void prefetch_tile(const Params<kMax>& p, int j, int item) {
  const Item& it = p.item[item];
  const int64_t r0 = (int64_t)(j - tile_begin(p, item)) * 16;
  const uint8_t* c = it.packed + r0 * (it.cols / 2);
  prefetch_range(c, c + (int64_t)16 * (it.cols / 2));
  const int64_t nbr = it.cols / kBlock;
  const int esz = it.kind == kPlain ? 4 : 1;
  const uint8_t* sc = static_cast<const uint8_t*>(it.scl) + r0 * nbr * esz;
  prefetch_range(sc, sc + 16 * nbr * esz);
}

// tiles prefetched ahead of the one a CTA starts: about 128 KB of codes
__device__ __forceinline__ int prefetch_distance(int cols) { return max(2, 131072 / (8 * cols)); }

template <int kMax, int kP0, int kP1, int kBook>
__global__ void __launch_bounds__(kThreads, 1) gemv_stream_kernel(const __grid_constant__ Params<kMax> p,
                                                                  unsigned* err) {
  extern __shared__ __align__(16) uint8_t smem[];
  // the pair table at the first 64 KB-aligned shared address; the partial slots and the unit table before it when
  // they fit there, else after it
  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);
  const uint32_t tpad = ((sbase + 65535u) & ~65535u) - sbase;
  uint8_t* table = smem + tpad;                                    // kPairTableBytes
  uint8_t* rest = tpad >= kRestBytes ? smem : table + kPairTableBytes;
  float* red = reinterpret_cast<float*>(rest);                     // [kSlots][kSlotFloats]
  float* unit = red + kSlots * kSlotFloats;                        // [2][256] dq units (E4M3, int8)
  __shared__ float code_s[16];
  __shared__ int red_count[kSlots];
  __shared__ int red_gen[kSlots];

  const int t_begin = p.cta_tile[blockIdx.x], t_end = p.cta_tile[blockIdx.x + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // The weights are read-only here: an L2 prefetch of the first tiles may run before the previous kernel in the
  // stream has finished (the register loads below come after griddepcontrol.wait and see its writes; L2 is the
  // point of coherence, so a prefetched line never hides a later write).
  if (threadIdx.x == 0 && t_begin < t_end) {
    int item = 0;
    while (t_begin >= p.tile_end[item]) ++item;
    const int dist = prefetch_distance(p.item[item].cols);
    for (int j = t_begin; j < min(t_begin + dist, t_end); ++j) {
      while (j >= p.tile_end[item]) ++item;
      prefetch_tile(p, j, item);
    }
  }
  pdl_launch_dependents();
  if (threadIdx.x < 16) code_s[threadIdx.x] = c_code_stream[kBook][threadIdx.x];
  if (threadIdx.x < kSlots) {
    red_count[threadIdx.x] = 0;
    red_gen[threadIdx.x] = 0;
  }
  for (int i = threadIdx.x; i < 512; i += kThreads) unit[i] = dq_unit(i & 255, i >> 8);
  __syncthreads();
  // pair table: entry v (code byte) of lane l at 256 v + 8 l holds (code[v >> 4], code[v & 15])
#pragma unroll
  for (int k = 0; k < kPairTableBytes / 16 / kThreads; ++k) {
    const int idx = threadIdx.x + k * kThreads;  // 16-byte pieces: two lanes' copies of one entry
    const float hi = code_s[idx >> 8], lo = code_s[(idx >> 4) & 15];
    *reinterpret_cast<float4*>(table + idx * 16) = make_float4(hi, lo, hi, lo);
  }
  __syncthreads();
  pdl_wait();

  const int g = lane >> 2, t = lane & 3;
  const int batch = p.batch;
  // prmt source for table addresses: byte 0 = 8 * lane, byte 1 = 0, bytes 2-3 = the table's 64 KB-aligned base
  const uint32_t lane_base = (uint32_t)(lane * 8) | (uint32_t)__cvta_generic_to_shared(table);
  const DecodeMul dm = decode_mul();
  constexpr int kG = kGroupSteps;  // steps per round-robin group

  // this warp's walk
  Walk wk;
  wk.j = t_begin;
  wk.item = 0;
  wk.gbase = 0;
  wk.G = warp;
  bool live = t_begin < t_end;
  if (live) {
    while (wk.j >= p.tile_end[wk.item]) ++wk.item;
    walk_tile<kG>(p, wk, g, t, batch);
    live = walk_locate<kG>(p, wk, t_end, g, t, batch);
  }

  auto next = [&]() {
    if (++wk.s < wk.send) return;
    const int j0 = wk.j;
    wk.G += kWarps;
    live = walk_locate<kG>(p, wk, t_end, g, t, batch);
    // the warp entering a tile with its first group prefetches the tile `prefetch_distance` ahead
    if (live && wk.j != j0 && wk.G == wk.gbase && lane == 0) {
      const int jp = wk.j + prefetch_distance(p.item[wk.item].cols);
      if (jp < t_end) {
        int item = wk.item;
        while (jp >= p.tile_end[item]) ++item;
        prefetch_tile(p, jp, item);
      }
    }
  };

  Step b0, b1;
  load_step(p, b0, wk, live, t_begin);
  if (live) next();
  load_step(p, b1, wk, live, t_begin);
  if (live) next();

  int cur_lj = -1, cur_info = 0;
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f}, acc2[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  int red_item = 0;

  // hand this warp's partial of tile cur_lj to the tile's reduction
  auto flush = [&]() {
    if (cur_lj < 0) return;
    const int slot = cur_lj & (kSlots - 1);
    // slot free: the reduction of tile cur_lj - kSlots is done (red_gen counts the slot's finished reductions)
    const int want = cur_lj / kSlots;
    auto gen_now = [&]() {
      int v;
      asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(&red_gen[slot])) : "memory");
      return v;
    };
    if (gen_now() < want) {
      const unsigned long long t0 = global_ns();
      while (gen_now() < want) {
        if (global_ns() - t0 > kWaitLimitNs) {
          atomicOr(err, kErrTimeout);
          break;
        }
      }
    }
    float* r = red + slot * kSlotFloats + (cur_info & 15) * 128;
    // accumulator fragment: c0 (row g, col 2t), c1 (g, 2t+1), c2 (g+8, 2t), c3 (g+8, 2t+1)
    *reinterpret_cast<float2*>(r + g * 8 + 2 * t) = make_float2(acc[0] + acc2[0], acc[1] + acc2[1]);
    *reinterpret_cast<float2*>(r + (g + 8) * 8 + 2 * t) = make_float2(acc[2] + acc2[2], acc[3] + acc2[3]);
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = acc2[i] = 0.0f;
    __syncwarp();
    const int tile = t_begin + cur_lj;
    while (tile >= p.tile_end[red_item]) ++red_item;
    const Item& it = p.item[red_item];
    const int parts = min(kWarps, tile_groups<kG>(it.cols));
    int last = 0;
    if (lane == 0) {  // release this warp's partial (ordered before lane 0 by __syncwarp); acquire the others'
      uint32_t old;
      asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;"
                   : "=r"(old) : "r"(smem_u32(&red_count[slot])) : "memory");
      last = (int)old == parts - 1;
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {  // the tile's last warp: partials in group order, then y
      __syncwarp();
      const int64_t rows = (int64_t)(p.tile_end[red_item] - tile_begin(p, red_item)) * 16;
      const int64_t row0 = (int64_t)(tile - tile_begin(p, red_item)) * 16;
      const float* rs = red + slot * kSlotFloats;
      for (int o = lane; o < 16 * batch; o += 32) {
        const int row = o & 15, b = o >> 4;
        float sum = 0.0f;
        for (int i = 0; i < parts; ++i) sum += *(volatile const float*)&rs[i * 128 + row * 8 + b];
        it.y[(int64_t)b * rows + row0 + row] = __float2bfloat16_rn(sum);
      }
      __syncwarp();
      if (lane == 0) {
        red_count[slot] = 0;
        asm volatile("red.release.cta.shared::cta.add.u32 [%0], 1;" ::"r"(smem_u32(&red_gen[slot])) : "memory");
      }
    }
  };

  // the step's reconstructed scales: plain absmax, or a^ = RN(RN(unit(q) * m) + mu)
  auto rebuild = [&](const Step& d, float& a0, float& a1) {
    const int kind = d.info >> 4;
    a0 = d.s0;
    a1 = d.s1;
    if (kind != kPlain) {
      const float* u = unit + (kind == kDqInt8 ? 256 : 0);
      a0 = dq_absmax(u[d.q & 255], d.s0, d.mu);
      a1 = dq_absmax(u[(d.q >> 8) & 255], d.s1, d.mu);
    }
  };
  auto prep = [&](Step& d) {
    if (d.lj >= 0) rebuild(d, d.a0, d.a1);
  };

  // decode + multiply one step into the accumulators
  auto consume = [&](const Step& d) {
    if (d.lj != cur_lj) {
      flush();
      cur_lj = d.lj;
    }
    cur_info = d.info;
    const float a0 = d.a0, a1 = d.a1;  // rebuilt one step ahead (prep)
    Table T0, T1;
    if (kP0 > 0) T0 = make_table<kBook>(a0);
    if (kP1 > 0) T1 = make_table<kBook>(a1);
    const uint32_t w0[8] = {d.w0[0].x, d.w0[0].y, d.w0[0].z, d.w0[0].w, d.w0[1].x, d.w0[1].y, d.w0[1].z, d.w0[1].w};
    const uint32_t w1[8] = {d.w1[0].x, d.w1[0].y, d.w1[0].z, d.w1[0].w, d.w1[1].x, d.w1[1].y, d.w1[1].z, d.w1[1].w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t e0[4], e1[4];
      if (j < kP0) decode_word(w0[j], T0, e0, dm); else table_decode(w0[j], a0, lane_base, e0);
      if (j < kP1) decode_word(w1[j], T1, e1, dm); else table_decode(w1[j], a1, lane_base, e1);
      const uint4 xv = __ldg(reinterpret_cast<const uint4*>(d.xp + 8 * j));
      float(&c)[4] = (j & 1) ? acc2 : acc;
      mma_bf16(c, e0[0], e1[0], e0[1], e1[1], xv.x, xv.y);
      mma_bf16(c, e0[2], e1[2], e0[3], e1[3], xv.z, xv.w);
    }
  };

  // two steps in flight: consume one while the next one's loads are outstanding (its scales, loaded a step
  // earlier, are rebuilt right after the current step)
  prep(b0);
  for (;;) {
    if (b0.lj < 0) break;
    consume(b0);
    prep(b1);
    load_step(p, b0, wk, live, t_begin);
    if (live) next();
    if (b1.lj < 0) break;
    consume(b1);
    prep(b0);
    load_step(p, b1, wk, live, t_begin);
    if (live) next();
  }
  flush();
}

template <int kMax, int kP0, int kP1, int kBook>
cudaError_t launch_variant(const Params<kMax>& p, int grid, unsigned* err, cudaStream_t stream) {
  constexpr size_t smem = kSmemBytes;
  static bool attr_done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {  // idempotent: a race only repeats the call
    const cudaError_t e = cudaFuncSetAttribute(gemv_stream_kernel<kMax, kP0, kP1, kBook>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const cudaError_t e = launch_pdl(gemv_stream_kernel<kMax, kP0, kP1, kBook>, dim3(grid), dim3(kThreads), smem, stream, p, err);
  count_launches(1);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int kMax>
cudaError_t launch_items(const GemvItem* items, int count, int batch, unsigned* err, cudaStream_t stream,
                         int num_sms) {
  Params<kMax> p = {};
  int64_t tiles = 0, work = 0;
  for (int i = 0; i < count; ++i) {
    const GemvItem& s = items[i];
    if (s.cols > INT32_MAX) return cudaErrorInvalidValue;
    tiles += s.rows / 16;
    work += s.rows / 16 * tile_groups<kGroupSteps>((int)s.cols);
    if (tiles > INT32_MAX) return cudaErrorInvalidValue;
    Item& d = p.item[i];
    d.packed = s.packed;
    d.cols = (int32_t)s.cols;
    d.x = static_cast<const __nv_bfloat16*>(s.x);
    d.y = static_cast<__nv_bfloat16*>(s.y);
    if (s.s.absmax != nullptr) {
      d.kind = kPlain;
      d.scl = s.s.absmax;
    } else {
      d.kind = s.s.dq_code == 0 ? kDqE4M3 : kDqInt8;
      d.scl = s.s.q;
      d.scale2 = s.s.scale;
      d.mean = s.s.mean;
    }
    p.tile_end[i] = (int32_t)tiles;
  }
  for (int i = count; i < kMax; ++i) p.tile_end[i] = (int32_t)tiles;  // the walks never pass the last item
  p.count = count;
  p.batch = batch;
  if (tiles == 0) return cudaSuccess;
  // one CTA per SM, at most one per tile; contiguous tile ranges of equal work (groups) to within one tile
  const int grid = (int)std::min<int64_t>(std::min(num_sms, kMaxCtas), tiles);
  p.cta_tile[0] = 0;
  int item = 0;
  int64_t wb = 0, t0 = 0;  // groups and tiles before item `item`
  for (int c = 1; c < grid; ++c) {
    const int64_t target = work * c / grid;
    for (;;) {
      const int64_t n = items[item].rows / 16, per = tile_groups<kGroupSteps>((int)items[item].cols);
      if (item == count - 1 || target < wb + n * per) {
        const int64_t k = std::min(n, std::max<int64_t>(0, (target - wb + per / 2) / per));
        p.cta_tile[c] = std::max<int32_t>(p.cta_tile[c - 1], (int32_t)(t0 + k));
        break;
      }
      wb += n * per;
      t0 += n;
      ++item;
    }
  }
  p.cta_tile[grid] = (int32_t)tiles;
  // Decode mix (words of row g through byte permutes; the other words, and all of row g + 8, through the pair
  // table), balancing the ALU pipe against shared-memory bandwidth: 6 of 16 at batch 1; at larger batches the
  // activation loads share the shared-memory/L1 data path, so 8 of 16
  const int book = items[0].s.book;
  for (int i = 1; i < count; ++i)
    if (items[i].s.book != book) return cudaErrorInvalidValue;  // one code book per launch
  // options 7: groups of 4 steps, scales rebuilt one step ahead, release/acquire hand-off of the partials (measured
  // 4-7% faster than none of them at 14336x4096, batch 1 and 8; hoisting a step's activation loads spilled)
  if (batch == 1)
    return book ? launch_variant<kMax, 6, 0, 1>(p, grid, err, stream)
                : launch_variant<kMax, 6, 0, 0>(p, grid, err, stream);
  return book ? launch_variant<kMax, 8, 0, 1>(p, grid, err, stream)
              : launch_variant<kMax, 8, 0, 0>(p, grid, err, stream);
}

}  // namespace

cudaError_t launch_gemv_items(const GemvItem* items, int count, int batch, unsigned* err, cudaStream_t stream,
                              int num_sms) {
  if (count < 1 || count > kMaxStreamItems || batch < 1 || batch > 8) return cudaErrorInvalidValue;
  if (count <= kMaxGroup) return launch_items<kMaxGroup>(items, count, batch, err, stream, num_sms);
  return launch_items<kMaxStreamItems>(items, count, batch, err, stream, num_sms);
}

}  // namespace nf4
