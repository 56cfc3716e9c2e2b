// gemm_sm100.cu -- prefill GEMM dispatcher.
#include "nf4_common.cuh"
#include "internal.h"

namespace nf4 {

size_t gemm_workspace_bytes(int64_t, int64_t, int64_t) { return 0; }

cudaError_t launch_gemm(const uint8_t* packed, const Scales& s, int64_t rows, int64_t cols, const void* x, int64_t m,
                        void* y, void*, unsigned*, cudaStream_t stream, int num_sms) {
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  auto* yb = static_cast<__nv_bfloat16*>(y);
  for (int64_t r = 0; r < m; r += 64) {
    const int chunk = (int)((m - r) < 64 ? (m - r) : 64);
    cudaError_t e = launch_gemv(packed, s, rows, cols, xb + r * cols, chunk, yb + r * rows, stream, num_sms);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace nf4
