// api.cu -- extern "C" entry points of libnf4 (declared in include/nf4.h).
// Host-side validation happens before any launch; kernels live in the other
// translation units (quantize.cu, double_quant.cu, dequantize.cu, gemv.cu,
// gemv_stream.cu, gemm_sm100.cu, gemm_dx_sm100.cu, lora_down.cu).
#include <atomic>
#include <mutex>

#include "../../include/nf4.h"
#include "internal.h"
#include "nf4_codebook.h"

namespace {

__device__ unsigned g_error_word;  // device-side error flags (nf4::kErrTimeout)

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  int cc_major = 0;
  unsigned* error_word = nullptr;
};

std::mutex g_mutex;
std::atomic<uint64_t> g_launches{0};
DeviceInfo g_info[kMaxDevices];

// Info of the current device, filled on first use.
nf4_status device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NF4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_info[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return NF4_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return NF4_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return NF4_ERR_CUDA;
    d.error_word = static_cast<unsigned*>(p);
    d.ready = true;
  }
  *out = d;
  return d.cc_major == 10 ? NF4_OK : NF4_ERR_ARCH;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

nf4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? NF4_OK : NF4_ERR_CUDA; }

bool level1_blocksize(int32_t b) { return b == 32 || b == 64 || b == 128 || b == 256; }

// Common checks of a weight descriptor; fills the kernel-side scale view.  The
// matmuls take 64-element blocks only; dequantization takes every level-1 size.
nf4_status check_weight(const nf4_weight* w, nf4::Scales* s, bool any_blocksize = false) {
  if (w == nullptr || w->packed == nullptr) return NF4_ERR_INVALID_ARG;
  if (w->rows < 0 || w->cols < 0) return NF4_ERR_INVALID_ARG;
  if (any_blocksize ? !level1_blocksize(w->blocksize) : w->blocksize != nf4::kBlock) return NF4_ERR_UNSUPPORTED;
  if (w->quant_type != NF4_QUANT_NF4 && w->quant_type != NF4_QUANT_FP4) return NF4_ERR_INVALID_ARG;
  if (!aligned(w->packed, 16)) return NF4_ERR_MISALIGNED;
  if (w->absmax != nullptr) {
    if (!aligned(w->absmax, 4)) return NF4_ERR_MISALIGNED;
    *s = nf4::Scales{w->absmax, nullptr, nullptr, nullptr, 0, w->quant_type};
    return NF4_OK;
  }
  if (w->absmax_q == nullptr || w->absmax_scale == nullptr || w->absmax_mean == nullptr) return NF4_ERR_INVALID_ARG;
  if (w->dq_blocksize != nf4::kDqBlock) return NF4_ERR_UNSUPPORTED;
  if (w->dq_code != NF4_DQ_E4M3 && w->dq_code != NF4_DQ_INT8) return NF4_ERR_INVALID_ARG;
  if (!aligned(w->absmax_scale, 4) || !aligned(w->absmax_mean, 4)) return NF4_ERR_MISALIGNED;
  *s = nf4::Scales{nullptr, w->absmax_q, w->absmax_scale, w->absmax_mean, w->dq_code, w->quant_type};
  return NF4_OK;
}

}  // namespace

namespace nf4 {
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace nf4

extern "C" {

uint64_t nf4_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char* nf4_status_string(nf4_status s) {
  switch (s) {
    case NF4_OK: return "NF4_OK";
    case NF4_ERR_INVALID_ARG: return "NF4_ERR_INVALID_ARG";
    case NF4_ERR_MISALIGNED: return "NF4_ERR_MISALIGNED";
    case NF4_ERR_UNSUPPORTED: return "NF4_ERR_UNSUPPORTED";
    case NF4_ERR_ARCH: return "NF4_ERR_ARCH";
    case NF4_ERR_CUDA: return "NF4_ERR_CUDA";
    case NF4_ERR_TIMEOUT: return "NF4_ERR_TIMEOUT";
  }
  return "NF4_ERR_UNKNOWN";
}

void nf4_code_table(float out[16]) {
  static const float code[16] = NF4_CODE_INIT;
  for (int i = 0; i < 16; ++i) out[i] = code[i];
}

size_t nf4_storage_bytes(int64_t n, int32_t blocksize, int32_t double_quant, int32_t dq_blocksize) {
  if (n <= 0 || blocksize <= 0) return 0;
  const size_t nb = (size_t)((n + blocksize - 1) / blocksize);
  size_t bytes = (size_t)((n + 1) / 2);
  if (!double_quant) return bytes + 4 * nb;
  if (dq_blocksize <= 0) return 0;
  return bytes + nb + 4 * ((nb + dq_blocksize - 1) / dq_blocksize) + 4;
}

size_t nf4_double_quant_workspace_bytes(int64_t /*nb*/) { return nf4::kDoubleQuantWorkspace; }

size_t nf4_gemm_workspace_bytes(const nf4_weight* w, int64_t m) {
  if (w == nullptr || w->rows <= 0 || w->cols <= 0 || m <= 0) return 0;
  return nf4::gemm_workspace_bytes(w->rows, w->cols, m);
}

size_t nf4_gemm_lora_workspace_bytes(const nf4_weight* w, int64_t m) {
  if (w == nullptr || w->rows <= 0 || w->cols <= 0 || m <= 0) return 0;
  return nf4::gemm_lora_workspace_bytes(w->rows, w->cols, m);
}

size_t nf4_gemm_dx_workspace_bytes(const nf4_weight* w, int64_t m) {
  if (w == nullptr || w->rows <= 0 || w->cols <= 0 || m <= 0) return 0;
  if (w->rows % 64 != 0 || w->cols % 128 != 0) return 0;
  return nf4::gemm_dx_workspace_bytes(w->rows, w->cols, m);
}

int32_t nf4_device_supported(void) {
  DeviceInfo d;
  return device_info(&d) == NF4_OK ? 1 : 0;
}

nf4_status nf4_quantize(const void* src, int32_t src_dtype, int64_t n, int32_t blocksize, uint8_t* packed_out,
                        float* absmax_out, nf4_stream_t stream) {
  return nf4_quantize_typed(src, src_dtype, n, blocksize, NF4_QUANT_NF4, packed_out, absmax_out, stream);
}

nf4_status nf4_quantize_typed(const void* src, int32_t src_dtype, int64_t n, int32_t blocksize, int32_t quant_type,
                              uint8_t* packed_out, float* absmax_out, nf4_stream_t stream) {
  if (n < 0) return NF4_ERR_INVALID_ARG;
  if (quant_type != NF4_QUANT_NF4 && quant_type != NF4_QUANT_FP4) return NF4_ERR_INVALID_ARG;
  if (src_dtype != NF4_F32 && src_dtype != NF4_BF16) return NF4_ERR_INVALID_ARG;
  if (!level1_blocksize(blocksize)) return NF4_ERR_UNSUPPORTED;
  if (n == 0) return NF4_OK;
  if (src == nullptr || packed_out == nullptr || absmax_out == nullptr) return NF4_ERR_INVALID_ARG;
  if (!aligned(src, 16) || !aligned(packed_out, 16) || !aligned(absmax_out, 4)) return NF4_ERR_MISALIGNED;
  DeviceInfo d;
  nf4_status st = device_info(&d);
  if (st != NF4_OK) return st;
  return from_cuda(nf4::launch_quantize(src, src_dtype == NF4_BF16, n, blocksize, packed_out, absmax_out, quant_type,
                                        reinterpret_cast<cudaStream_t>(stream), d.num_sms));
}

static_assert(NF4_QUANT_MANY_MAX == nf4::kQuantManyMax, "array limit");

nf4_status nf4_quantize_many(const void* const* src, const int64_t* n, int32_t count, int32_t src_dtype,
                             int32_t blocksize, int32_t quant_type, uint8_t* const* packed_out,
                             float* const* absmax_out, nf4_stream_t stream) {
  if (count < 1 || count > NF4_QUANT_MANY_MAX) return NF4_ERR_INVALID_ARG;
  if (src == nullptr || n == nullptr || packed_out == nullptr || absmax_out == nullptr) return NF4_ERR_INVALID_ARG;
  if (quant_type != NF4_QUANT_NF4 && quant_type != NF4_QUANT_FP4) return NF4_ERR_INVALID_ARG;
  if (src_dtype != NF4_F32 && src_dtype != NF4_BF16) return NF4_ERR_INVALID_ARG;
  if (!level1_blocksize(blocksize)) return NF4_ERR_UNSUPPORTED;
  // every tensor is checked before anything is launched; empty ones are left out
  static thread_local nf4::QuantManyParams p;  // 10 KB: kept off the stack
  p.count = 0;
  for (int32_t i = 0; i < count; ++i) {
    if (n[i] < 0) return NF4_ERR_INVALID_ARG;
    if (n[i] == 0) continue;
    if (src[i] == nullptr || packed_out[i] == nullptr || absmax_out[i] == nullptr) return NF4_ERR_INVALID_ARG;
    if (!aligned(src[i], 16) || !aligned(packed_out[i], 16) || !aligned(absmax_out[i], 4))
      return NF4_ERR_MISALIGNED;
    nf4::QuantItem& it = p.item[p.count++];
    it.src = src[i];
    it.packed = packed_out[i];
    it.absmax = absmax_out[i];
    it.n = n[i];
  }
  if (p.count == 0) return NF4_OK;
  DeviceInfo d;
  nf4_status st = device_info(&d);
  if (st != NF4_OK) return st;
  return from_cuda(nf4::launch_quantize_many(p, src_dtype == NF4_BF16, blocksize, quant_type,
                                             reinterpret_cast<cudaStream_t>(stream), d.num_sms));
}

nf4_status nf4_double_quant(const float* absmax, int64_t nb, int32_t dq_blocksize, int32_t dq_code, uint8_t* q_out,
                            float* scale_out, float* mean_out, void* workspace, size_t workspace_bytes,
                            nf4_stream_t stream) {
  if (nb < 0 || nb > NF4_DQ_MAX_NB) return NF4_ERR_INVALID_ARG;
  if (dq_code != NF4_DQ_E4M3 && dq_code != NF4_DQ_INT8) return NF4_ERR_INVALID_ARG;
  if (dq_blocksize != nf4::kDqBlock) return NF4_ERR_UNSUPPORTED;
  if (nb == 0) return NF4_OK;
  if (absmax == nullptr || q_out == nullptr || scale_out == nullptr || mean_out == nullptr || workspace == nullptr)
    return NF4_ERR_INVALID_ARG;
  if (workspace_bytes < nf4::kDoubleQuantWorkspace) return NF4_ERR_INVALID_ARG;
  if (!aligned(absmax, 16) || !aligned(q_out, 16) || !aligned(scale_out, 4) || !aligned(mean_out, 4) ||
      !aligned(workspace, 16))
    return NF4_ERR_MISALIGNED;
  DeviceInfo d;
  nf4_status st = device_info(&d);
  if (st != NF4_OK) return st;
  return from_cuda(nf4::launch_double_quant(absmax, nb, dq_code, q_out, scale_out, mean_out, workspace, false,
                                            d.error_word, reinterpret_cast<cudaStream_t>(stream), d.num_sms));
}

static_assert(NF4_DQ_MANY_MAX == nf4::kDqManyMax, "array limit");

size_t nf4_double_quant_many_workspace_bytes(int32_t count) {
  return count < 1 || count > NF4_DQ_MANY_MAX ? 0 : (size_t)count * nf4::kDqManyRecord;
}

nf4_status nf4_double_quant_many(const float* const* absmax, const int64_t* nb, int32_t count, int32_t dq_blocksize,
                                 int32_t dq_code, uint8_t* const* q_out, float* const* scale_out,
                                 float* const* mean_out, void* workspace, size_t workspace_bytes,
                                 nf4_stream_t stream) {
  if (count < 1 || count > NF4_DQ_MANY_MAX) return NF4_ERR_INVALID_ARG;
  if (absmax == nullptr || nb == nullptr || q_out == nullptr || scale_out == nullptr || mean_out == nullptr)
    return NF4_ERR_INVALID_ARG;
  if (dq_code != NF4_DQ_E4M3 && dq_code != NF4_DQ_INT8) return NF4_ERR_INVALID_ARG;
  if (dq_blocksize != nf4::kDqBlock) return NF4_ERR_UNSUPPORTED;
  if (workspace == nullptr || workspace_bytes < nf4_double_quant_many_workspace_bytes(count))
    return NF4_ERR_INVALID_ARG;
  if (!aligned(workspace, 16)) return NF4_ERR_MISALIGNED;
  // every array is checked before anything is launched; empty ones are left out (their mean_out stays unset)
  static thread_local nf4::DqManyParams p;  // 14 KB: kept off the stack
  p.count = 0;
  p.total = 0;
  p.groups = 0;
  for (int32_t i = 0; i < count; ++i) {
    if (nb[i] < 0 || nb[i] > NF4_DQ_MAX_NB) return NF4_ERR_INVALID_ARG;
    if (nb[i] == 0) continue;
    if (absmax[i] == nullptr || q_out[i] == nullptr || scale_out[i] == nullptr || mean_out[i] == nullptr)
      return NF4_ERR_INVALID_ARG;
    if (!aligned(absmax[i], 16) || !aligned(q_out[i], 16) || !aligned(scale_out[i], 4) || !aligned(mean_out[i], 4))
      return NF4_ERR_MISALIGNED;
    nf4::DqItem& it = p.item[p.count++];
    it.a = absmax[i];
    it.q = q_out[i];
    it.scale = scale_out[i];
    it.mean = mean_out[i];
    it.nb = nb[i];
    it.e0 = p.total;
    it.g0 = p.groups;
    p.total += nb[i];
    p.groups += (nb[i] + nf4::kDqBlock - 1) / nf4::kDqBlock;
  }
  if (p.count == 0) return NF4_OK;
  DeviceInfo d;
  nf4_status st = device_info(&d);
  if (st != NF4_OK) return st;
  return from_cuda(nf4::launch_double_quant_many(p, dq_code, workspace, reinterpret_cast<cudaStream_t>(stream),
                                                 d.num_sms));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Double quantization with library-owned scratch (no caller workspace).
// The scratch is a file-scope device array; host code only ever uses the
// device address looked up below, never the symbol itself (in host code the
// symbol's name is a host-side stand-in, not a device address).
namespace {

constexpr size_t kNoAllocScratchBytes = 256;  // one exact-sum record (limbs + barrier count)
static_assert(kNoAllocScratchBytes >= nf4::kDoubleQuantWorkspace, "scratch too small");
__device__ __align__(256) unsigned char g_dq_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices];  // device address of g_dq_scratch, per device

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached.
nf4_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NF4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dq_scratch) != cudaSuccess || p == nullptr) return NF4_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return NF4_OK;
}

}  // namespace

extern "C" {

nf4_status nf4_double_quant_noalloc(const float* absmax, int64_t nb, int32_t dq_blocksize, int32_t dq_code,
                                    uint8_t* q_out, float* scale_out, float* mean_out, nf4_stream_t stream) {
  if (nb < 0 || nb > NF4_DQ_NOALLOC_MAX_NB) return NF4_ERR_INVALID_ARG;
  if (dq_code != NF4_DQ_E4M3 && dq_code != NF4_DQ_INT8) return NF4_ERR_INVALID_ARG;
  if (dq_blocksize != nf4::kDqBlock) return NF4_ERR_UNSUPPORTED;
  if (nb == 0) return NF4_OK;
  if (absmax == nullptr || q_out == nullptr || scale_out == nullptr || mean_out == nullptr)
    return NF4_ERR_INVALID_ARG;
  if (!aligned(absmax, 16) || !aligned(q_out, 16) || !aligned(scale_out, 4) || !aligned(mean_out, 4))
    return NF4_ERR_MISALIGNED;
  DeviceInfo d;
  nf4_status st = device_info(&d);
  if (st != NF4_OK) return st;
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != NF4_OK) return st;
  // the launcher clears the scratch on `stream` before the kernel reads it
  return from_cuda(nf4::launch_double_quant(absmax, nb, dq_code, q_out, scale_out, mean_out, scratch, true,
                                            d.error_word, reinterpret_cast<cudaStream_t>(stream), d.num_sms));
}

nf4_status nf4_dequantize(const nf4_weight* w, void* out, int32_t out_dtype, nf4_stream_t stream) {
  nf4::Scales s;
  nf4_status st = check_weight(w, &s, true);
  if (st != NF4_OK) return st;
  if (out_dtype != NF4_F32 && out_dtype != NF4_BF16) return NF4_ERR_INVALID_ARG;
  const int64_t n = w->rows * w->cols;
  if (n == 0) return NF4_OK;
  if (out == nullptr) return NF4_ERR_INVALID_ARG;
  if (!aligned(out, 16)) return NF4_ERR_MISALIGNED;
  DeviceInfo d;
  if ((st = device_info(&d)) != NF4_OK) return st;
  return from_cuda(nf4::launch_dequantize(w->packed, s, n, w->blocksize, out, out_dtype == NF4_BF16,
                                          reinterpret_cast<cudaStream_t>(stream), d.num_sms));
}

nf4_status nf4_gemv(const nf4_weight* w, const void* x, int32_t batch, void* y, nf4_stream_t stream) {
  nf4::Scales s;
  nf4_status st = check_weight(w, &s);
  if (st != NF4_OK) return st;
  if (batch < 1 || batch > 8) return NF4_ERR_INVALID_ARG;
  if (w->cols % nf4::kBlock != 0 || w->rows % 16 != 0) return NF4_ERR_UNSUPPORTED;
  if (w->rows == 0 || w->cols == 0) return NF4_OK;
  if (x == nullptr || y == nullptr) return NF4_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 4)) return NF4_ERR_MISALIGNED;
  DeviceInfo d;
  if ((st = device_info(&d)) != NF4_OK) return st;
  return from_cuda(nf4::launch_gemv(w->packed, s, w->rows, w->cols, x, batch, y, d.error_word,
                                    reinterpret_cast<cudaStream_t>(stream), d.num_sms));
}

nf4_status nf4_gemv_grouped(const nf4_weight* const* ws, int32_t count, const void* x, int32_t batch, void* const* ys,
                            nf4_stream_t stream) {
  if (ws == nullptr || ys == nullptr || count < 1 || count > nf4::kMaxGroup) return NF4_ERR_INVALID_ARG;
  if (batch < 1 || batch > 8) return NF4_ERR_INVALID_ARG;
  nf4::Scales s[nf4::kMaxGroup];
  const uint8_t* packed[nf4::kMaxGroup];
  int64_t rows[nf4::kMaxGroup];
  void* y[nf4::kMaxGroup];
  int n = 0;
  for (int i = 0; i < count; ++i) {
    nf4_status st = check_weight(ws[i], &s[n]);
    if (st != NF4_OK) return st;
    const nf4_weight* w = ws[i];
    if (w->cols != ws[0]->cols || (w->absmax == nullptr) != (ws[0]->absmax == nullptr) ||
        w->quant_type != ws[0]->quant_type)
      return NF4_ERR_INVALID_ARG;
    if (w->cols % nf4::kBlock != 0 || w->rows % 16 != 0) return NF4_ERR_UNSUPPORTED;
    if (w->rows == 0) continue;  // nothing to compute for an empty weight
    if (ys[i] == nullptr) return NF4_ERR_INVALID_ARG;
    if (!aligned(ys[i], 4)) return NF4_ERR_MISALIGNED;
    packed[n] = w->packed;
    rows[n] = w->rows;
    y[n] = ys[i];
    ++n;
  }
  if (n == 0 || ws[0]->cols == 0) return NF4_OK;
  if (x == nullptr) return NF4_ERR_INVALID_ARG;
  if (!aligned(x, 16)) return NF4_ERR_MISALIGNED;
  DeviceInfo d;
  nf4_status st = device_info(&d);
  if (st != NF4_OK) return st;
  return from_cuda(nf4::launch_gemv_group(packed, s, rows, n, ws[0]->cols, x, batch, y, d.error_word,
                                          reinterpret_cast<cudaStream_t>(stream), d.num_sms));
}

nf4_status nf4_gemv_stream(const nf4_weight* ws, const void* const* xs, void* const* ys, int32_t count, int32_t batch,
                           nf4_stream_t stream) {
  if (ws == nullptr || xs == nullptr || ys == nullptr || count < 1 || count > NF4_GEMV_STREAM_MAX)
    return NF4_ERR_INVALID_ARG;
  if (batch < 1 || batch > 8) return NF4_ERR_INVALID_ARG;
  static_assert(NF4_GEMV_STREAM_MAX <= nf4::kMaxStreamItems, "stream capacity");
  nf4::GemvItem items[NF4_GEMV_STREAM_MAX];
  int n = 0;
  for (int i = 0; i < count; ++i) {
    const nf4_weight* w = &ws[i];
    nf4::Scales s;
    nf4_status st = check_weight(w, &s);
    if (st != NF4_OK) return st;
    if (w->quant_type != ws[0].quant_type) return NF4_ERR_INVALID_ARG;  // one code book per launch
    if (w->cols % nf4::kBlock != 0 || w->rows % 16 != 0) return NF4_ERR_UNSUPPORTED;
    if (w->rows == 0 || w->cols == 0) continue;  // nothing to compute for an empty weight
    if (xs[i] == nullptr || ys[i] == nullptr) return NF4_ERR_INVALID_ARG;
    if (!aligned(xs[i], 16) || !aligned(ys[i], 4)) return NF4_ERR_MISALIGNED;
    items[n++] = nf4::GemvItem{w->packed, s, xs[i], ys[i], w->rows, w->cols};
  }
  if (n == 0) return NF4_OK;
  DeviceInfo d;
  nf4_status st = device_info(&d);
  if (st != NF4_OK) return st;
  return from_cuda(nf4::launch_gemv_items(items, n, batch, d.error_word, reinterpret_cast<cudaStream_t>(stream),
                                          d.num_sms));
}

nf4_status nf4_gemm(const nf4_weight* w, const void* x, int64_t m, void* y, void* workspace, size_t workspace_bytes,
                    nf4_stream_t stream) {
  nf4::Scales s;
  nf4_status st = check_weight(w, &s);
  if (st != NF4_OK) return st;
  if (m < 0) return NF4_ERR_INVALID_ARG;
  if (w->cols % nf4::kBlock != 0 || w->rows % 128 != 0) return NF4_ERR_UNSUPPORTED;
  if (m == 0 || w->rows == 0 || w->cols == 0) return NF4_OK;
  if (x == nullptr || y == nullptr) return NF4_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16)) return NF4_ERR_MISALIGNED;
  const size_t need = nf4::gemm_workspace_bytes(w->rows, w->cols, m);
  if (workspace_bytes < need || (need > 0 && workspace == nullptr)) return NF4_ERR_INVALID_ARG;
  if (need > 0 && !aligned(workspace, 16)) return NF4_ERR_MISALIGNED;
  DeviceInfo d;
  if ((st = device_info(&d)) != NF4_OK) return st;
  return from_cuda(nf4::launch_gemm(w->packed, s, w->rows, w->cols, x, m, y, workspace, d.error_word,
                                    reinterpret_cast<cudaStream_t>(stream), d.num_sms));
}

nf4_status nf4_gemm_lora(const nf4_weight* w, const nf4_lora* lora, const void* x, int64_t m, void* y,
                         void* workspace, size_t workspace_bytes, nf4_stream_t stream) {
  nf4::Scales s;
  nf4_status st = check_weight(w, &s);
  if (st != NF4_OK) return st;
  if (w->quant_type != NF4_QUANT_NF4) return NF4_ERR_UNSUPPORTED;  // NF4 codes only
  if (m < 0 || lora == nullptr) return NF4_ERR_INVALID_ARG;
  if (lora->r != 16 && lora->r != 32) return NF4_ERR_UNSUPPORTED;
  if (!(lora->scale == lora->scale) || lora->scale - lora->scale != 0.0f) return NF4_ERR_INVALID_ARG;  // finite
  if (w->cols % nf4::kBlock != 0 || w->rows % 128 != 0) return NF4_ERR_UNSUPPORTED;
  if (m == 0 || w->rows == 0 || w->cols == 0) return NF4_OK;
  if (x == nullptr || y == nullptr || lora->down == nullptr || lora->up == nullptr || workspace == nullptr)
    return NF4_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(lora->down, 16) || !aligned(lora->up, 16) ||
      !aligned(workspace, 16))
    return NF4_ERR_MISALIGNED;
  if (workspace_bytes < nf4::gemm_lora_workspace_bytes(w->rows, w->cols, m)) return NF4_ERR_INVALID_ARG;
  DeviceInfo d;
  if ((st = device_info(&d)) != NF4_OK) return st;
  return from_cuda(nf4::launch_gemm_lora(w->packed, s, w->rows, w->cols, x, m, lora->down, lora->up, lora->r,
                                         lora->scale, y, workspace, d.error_word,
                                         reinterpret_cast<cudaStream_t>(stream), d.num_sms));
}

nf4_status nf4_gemm_dx(const nf4_weight* w, const void* dy, int64_t m, void* dx, void* workspace,
                       size_t workspace_bytes, nf4_stream_t stream) {
  nf4::Scales s;
  nf4_status st = check_weight(w, &s);
  if (st != NF4_OK) return st;
  if (w->quant_type != NF4_QUANT_NF4) return NF4_ERR_UNSUPPORTED;  // NF4 codes only
  if (m < 0) return NF4_ERR_INVALID_ARG;
  if (w->rows % 64 != 0 || w->cols % 128 != 0) return NF4_ERR_UNSUPPORTED;
  if (m == 0 || w->rows == 0 || w->cols == 0) return NF4_OK;
  if (dy == nullptr || dx == nullptr) return NF4_ERR_INVALID_ARG;
  if (!aligned(dy, 16) || !aligned(dx, 16)) return NF4_ERR_MISALIGNED;
  const size_t need = nf4::gemm_dx_workspace_bytes(w->rows, w->cols, m);
  if (workspace_bytes < need || (need > 0 && workspace == nullptr)) return NF4_ERR_INVALID_ARG;
  if (need > 0 && !aligned(workspace, 16)) return NF4_ERR_MISALIGNED;
  DeviceInfo d;
  if ((st = device_info(&d)) != NF4_OK) return st;
  return from_cuda(nf4::launch_gemm_dx(w->packed, s, w->rows, w->cols, dy, m, dx, workspace, d.error_word,
                                       reinterpret_cast<cudaStream_t>(stream), d.num_sms));
}

nf4_status nf4_check_device_error(nf4_stream_t stream) {
  DeviceInfo d;
  nf4_status st = device_info(&d);
  if (st != NF4_OK) return st;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return NF4_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpy(&word, d.error_word, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess) return NF4_ERR_CUDA;
  if (word != 0) {
    const unsigned zero = 0;
    if (cudaMemcpy(d.error_word, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return NF4_ERR_CUDA;
    return NF4_ERR_TIMEOUT;
  }
  return NF4_OK;
}

nf4_status nf4_selftest_wait_timeout(nf4_stream_t stream) {
  DeviceInfo d;
  nf4_status st = device_info(&d);
  if (st != NF4_OK) return st;
  return from_cuda(nf4::launch_wait_timeout(d.error_word, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
