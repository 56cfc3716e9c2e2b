// internal.h -- launchers behind the C ABI (see include/nf4.h for semantics).
// Arguments are validated by the callers in api.cu; launchers only size grids.
#pragma once
#include <cuda_runtime.h>
#include <cstdint>

namespace nf4 {

// Launch with programmatic stream serialization: the kernel may start while the
// previous kernel in the stream finishes; it waits for it (griddepcontrol.wait)
// before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

constexpr int kBlock = 64;      // level-1 block (elements per absmax)
constexpr int kDqBlock = 256;   // level-2 block (absmax values per second-level scale)

// Level-1 scales as the kernels see them: plain fp32 absmax, or the
// double-quantized record (8-bit codes + second-level block absmax + mean).
// count of kernels launched (read by nf4_kernel_launches)
void count_launches(int n);

struct Scales {
  const float* absmax;   // non-null: plain scales
  const uint8_t* q;      // double-quantized codes
  const float* scale;    // second-level block absmax
  const float* mean;     // device pointer to the removed mean
  int dq_code;           // 0 = E4M3, 1 = int8
  int book;              // 4-bit code book: 0 = NF4, 1 = FP4 (E2M1 / 6)
};

// blocksize 32, 64, 128 or 256
cudaError_t launch_quantize(const void* src, bool bf16, int64_t n, int blocksize, uint8_t* packed, float* absmax,
                            int book, cudaStream_t stream, int num_sms);

// several tensors of one dtype, block size and code book in one launch (w0 and iters are filled by the launcher)
constexpr int kQuantManyMax = 256;
struct QuantItem {
  const void* src;  // n elements, 16-byte aligned
  uint8_t* packed;  // ceil(n / 2)
  float* absmax;    // ceil(n / blocksize)
  int64_t n;        // >= 1
  int64_t w0;       // first warp iteration of this tensor in the launch's sequence
};
struct QuantManyParams {
  QuantItem item[kQuantManyMax];
  int32_t count;  // >= 1
  int64_t iters;  // warp iterations of all tensors
};
cudaError_t launch_quantize_many(QuantManyParams& p, bool bf16, int blocksize, int book, cudaStream_t stream,
                                 int num_sms);

// workspace: zero before its first use, left ready by every completed call; `clear` zeroes it first
cudaError_t launch_double_quant(const float* absmax, int64_t nb, int dq_code, uint8_t* q, float* scale,
                                float* mean, void* workspace, bool clear, unsigned* err, cudaStream_t stream,
                                int num_sms);
constexpr size_t kDoubleQuantWorkspace = 256;

// double quantization of several absmax arrays in two launches (one exact-sum record per tensor in the workspace)
constexpr int kDqManyMax = 256;
constexpr size_t kDqManyRecord = 128;  // workspace bytes per tensor
struct DqItem {
  const float* a;  // absmax [nb], 16-byte aligned
  uint8_t* q;      // codes [nb]
  float* scale;    // [ceil(nb / 256)]
  float* mean;     // [1]
  int64_t nb;      // >= 1
  int64_t e0;      // first element of this array in the concatenation of all of them
  int64_t g0;      // first 256-block likewise
};
struct DqManyParams {
  DqItem item[kDqManyMax];
  int32_t count;   // >= 1
  int64_t total;   // sum of nb
  int64_t groups;  // sum of ceil(nb / 256)
};
cudaError_t launch_double_quant_many(const DqManyParams& p, int dq_code, void* workspace, cudaStream_t stream,
                                     int num_sms);

// blocksize 32, 64, 128 or 256
cudaError_t launch_dequantize(const uint8_t* packed, const Scales& s, int64_t n, int blocksize, void* out,
                              bool out_bf16, cudaStream_t stream, int num_sms);

// one CTA per 16-row tile (gemv.cu); batch up to 64
cudaError_t launch_gemv(const uint8_t* packed, const Scales& s, int64_t rows, int64_t cols, const void* x,
                        int batch, void* y, unsigned* err, cudaStream_t stream, int num_sms);

// several weights (same cols and scale kind) on one input in one launch, count <= kMaxGroup
constexpr int kMaxGroup = 4;
cudaError_t launch_gemv_group(const uint8_t* const* packed, const Scales* s, const int64_t* rows, int count,
                              int64_t cols, const void* x, int batch, void* const* y, unsigned* err,
                              cudaStream_t stream, int num_sms);

// one GEMV of the persistent stream: weight [rows, cols] (rows % 16 == 0, cols % 64 == 0), its input x [batch, cols]
// and output y [batch, rows]; up to kMaxStreamItems of them in one launch, batch 1..8
struct GemvItem {
  const uint8_t* packed;
  Scales s;
  const void* x;
  void* y;
  int64_t rows, cols;
};
constexpr int kMaxStreamItems = 256;
cudaError_t launch_gemv_items(const GemvItem* items, int count, int batch, unsigned* err, cudaStream_t stream,
                              int num_sms);

size_t gemm_workspace_bytes(int64_t rows, int64_t cols, int64_t m);
cudaError_t launch_gemm(const uint8_t* packed, const Scales& s, int64_t rows, int64_t cols, const void* x,
                        int64_t m, void* y, void* workspace, unsigned* err, cudaStream_t stream, int num_sms);

// 4-bit matmul plus a low-rank adapter: T = scale * X . A^T as a bf16 pair [hi | lo] into the first bytes of
// the workspace ([m, 64] bf16), then the GEMM with one adapter stage per output tile (r in {16, 32})
cudaError_t launch_lora_down(const void* x, const void* a, int64_t m, int64_t cols, int r, float scale, void* t,
                             cudaStream_t stream);
size_t gemm_lora_workspace_bytes(int64_t rows, int64_t cols, int64_t m);
cudaError_t launch_gemm_lora(const uint8_t* packed, const Scales& s, int64_t rows, int64_t cols, const void* x,
                             int64_t m, const void* lora_down, const void* lora_up, int lora_r, float lora_scale,
                             void* y, void* workspace, unsigned* err, cudaStream_t stream, int num_sms);

// input gradient dX = dY . Wc (rows % 64 == 0, cols % 128 == 0)
size_t gemm_dx_workspace_bytes(int64_t rows, int64_t cols, int64_t m);
cudaError_t launch_gemm_dx(const uint8_t* packed, const Scales& s, int64_t rows, int64_t cols, const void* dy,
                           int64_t m, void* dx, void* workspace, unsigned* err, cudaStream_t stream, int num_sms);

// failure-path self-test: a bounded wait that runs out (see selftest.cu)
cudaError_t launch_wait_timeout(unsigned* err, cudaStream_t stream);

}  // namespace nf4
