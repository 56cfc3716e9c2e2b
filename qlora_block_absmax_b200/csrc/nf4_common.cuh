// nf4_common.cuh -- device helpers shared by the libnf4 kernels (sm_100a).
//
// Numerics follow the bitsandbytes / QLoRA pages: blockwise absmax scaling and
// nearest-code rounding ("bitsandbytes", ozercemkelahmet.com/tools, "How it
// works" Steps 1-5), the NF4 code book ("How NF4 works"), double quantization
// of the scales ("Double quantization"; "bitsandbytes quantization tutorial",
// mljourney.com, "How NF4 Works").  Every rounding the method fixes is written
// with an explicit round-to-nearest intrinsic (__fmul_rn, __fdiv_rn, ...) so the
// compiler cannot contract it into a fused multiply-add.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "internal.h"
#include "nf4_codebook.h"

namespace nf4 {

constexpr float kE4M3Top = 448.0f;
constexpr float kInt8Top = 127.0f;

// error word bits set by device code (read back by nf4_check_device_error)
constexpr unsigned kErrTimeout = 1u;

// wall-clock bound of every device-side wait (nanoseconds)
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// two fp32 -> packed bf16x2 (round to nearest even); `lo` lands in bits 0..15
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ float bf16_lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// two fp32 -> two E4M3 bytes (round to nearest even, saturating to +-448);
// `lo` lands in bits 0..7
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  unsigned short d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

// E4M3 byte -> fp32 (exact, through the hardware fp8 -> f16 conversion)
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h2;
  unsigned short in = (unsigned short)(code & 0xffu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu)));
}

// value of one second-level code, back in [-1, 1]: RN(dec(q) / Q)
__device__ __forceinline__ float dq_unit(uint32_t q, int dq_code) {
  if (dq_code == 0) return __fdiv_rn(e4m3_to_f32(q), kE4M3Top);
  return __fdiv_rn((float)(int8_t)(uint8_t)q, kInt8Top);
}

// Reconstructed level-1 scale: a^ = RN(RN(unit * m) + mu)
__device__ __forceinline__ float dq_absmax(float unit, float m, float mu) {
  return __fadd_rn(__fmul_rn(unit, m), mu);
}

// ---------------------------------------------------------------- mbarrier / async proxy

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of a barrier, giving up after kWaitLimitNs of wall
// clock: on timeout the error word gets kErrTimeout and the function returns
// false so the caller can leave its loop instead of hanging the GPU.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, unsigned* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) break;
  }
  if (err) atomicOr(err, kErrTimeout);
  return false;
}

// Programmatic dependent launch.  Every kernel of the library signals at entry
// that the next kernel in the stream may start its own set-up, and waits for
// the previous kernel (its completion and memory) before its first access to
// global memory; without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace nf4
