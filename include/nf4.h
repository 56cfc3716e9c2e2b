/*
 * nf4.h -- C ABI of libnf4: blockwise NF4 4-bit weight quantization with double
 * quantization of the absmax constants, dequantization, and the 4-bit-weight x
 * bf16-activation matmul that dequantizes on the fly (GEMV for decode, also
 * grouped over weights that share an input; GEMM for prefill, also with a
 * low-rank adapter in the same accumulator; and the GEMM's input gradient
 * through the frozen weight), for NVIDIA B200 (sm_100a).
 *
 * Method sources (web pages on bitsandbytes / QLoRA):
 *   [bnb-tools] "bitsandbytes" (ozercemkelahmet.com/tools/bitsandbytes):
 *               "How it works" Steps 1-5, "How NF4 works", "Double quantization",
 *               "A worked example", "Fine-tuning with adapters on a 4-bit
 *               model", "Strengths and limitations".
 *   [bnb-tut]   "bitsandbytes quantization tutorial: 4-bit and 8-bit models"
 *               (mljourney.com): "4-bit Loading with NF4", "How NF4 Works",
 *               "QLoRA: Fine-Tuning a 4-bit Model".
 *
 * Conventions for every entry point:
 *   - Memory: all buffers are allocated and owned by the caller; the library
 *     allocates nothing.  "device" pointers must point to memory of the
 *     current CUDA device; "host" pointers to host memory.
 *   - Execution: work is enqueued asynchronously on `stream` (a cudaStream_t;
 *     NULL = legacy default stream).  Arguments are validated on the host
 *     first; on any error nothing is launched and no buffer is touched.
 *   - Alignment: device pointers must be 16-byte aligned unless stated
 *     otherwise (NF4_ERR_MISALIGNED).
 *   - Sizes: element counts are int64; 0 is valid and launches nothing.
 *   - Inputs must be finite; NaN or Inf inputs give unspecified codes.
 *   - No in-place operation: outputs must not overlap inputs.
 *   - Errors: functions return an nf4_status and never throw or abort.
 *     NF4_ERR_CUDA carries a launch failure; device-side waits that exceed
 *     their bound set an error word read by nf4_check_device_error().
 *   - Thread safety: every function is reentrant; concurrent calls on
 *     different streams are independent.
 */
#ifndef NF4_H
#define NF4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NF4_API __attribute__((visibility("default")))
#else
#define NF4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *nf4_stream_t; /* same type as cudaStream_t */

typedef enum {
  NF4_OK = 0,
  NF4_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad enum, short workspace */
  NF4_ERR_MISALIGNED = 2,  /* a pointer breaks the stated alignment */
  NF4_ERR_UNSUPPORTED = 3, /* a valid but unimplemented configuration */
  NF4_ERR_ARCH = 4,        /* current device is not sm_100 (B200 class) */
  NF4_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
  NF4_ERR_TIMEOUT = 6      /* a device-side wait gave up (see nf4_check_device_error) */
} nf4_status;

typedef enum { NF4_F32 = 0, NF4_BF16 = 1 } nf4_dtype;

/* 8-bit code of the double-quantized absmax constants.
 * NF4_DQ_E4M3: OCP FP8 E4M3 ("float8", [bnb-tut] "How NF4 Works"), top code 448.
 * NF4_DQ_INT8: linear int8 -127..127, round half away from zero ([bnb-tools]
 *              "A worked example"), top code 127. */
typedef enum { NF4_DQ_E4M3 = 0, NF4_DQ_INT8 = 1 } nf4_dq_code;

/* The 4-bit code book ([bnb-tools] "What it is": 4-bit layers in NF4 or FP4;
 * "Glossary", the FP4 entry; [bnb-tut] "4-bit Loading with NF4").
 * NF4_QUANT_NF4: the 16 NF4 levels (normal quantiles scaled to [-1, 1],
 *                ascending, index 7 = 0).
 * NF4_QUANT_FP4: the 4-bit float E2M1 (sign, 2 exponent bits with bias 1,
 *                1 mantissa bit) divided by 6 so that +-6 maps to +-1; the
 *                4-bit code is the E2M1 bit pattern (8 = -0).  Nearest level
 *                with ties to the even mantissa bit; a zero result keeps the
 *                sign of the value; an all-zero block and an odd tail's
 *                partner are +0. */
typedef enum { NF4_QUANT_NF4 = 0, NF4_QUANT_FP4 = 1 } nf4_quant_type;

/* A quantized weight W of shape [rows, cols] (row-major, rows = output
 * features N, cols = input features K), flattened for quantization so the
 * level-1 blocks run along a row.  All pointers are device pointers.
 *   packed        ceil(rows*cols/2) bytes, two codes per byte, element 2j in
 *                 the high nibble of byte j ([bnb-tools] Step 4)
 *   absmax        nb = ceil(rows*cols/blocksize) fp32 block scales, or NULL
 *                 when the weight is double-quantized
 *   absmax_q      nb 8-bit codes of the mean-removed scales (double quant)
 *   absmax_scale  ceil(nb/dq_blocksize) fp32 second-level block absmax values
 *   absmax_mean   1 fp32: the mean removed before second-level quantization
 *   blocksize     level-1 block size: 32, 64, 128 or 256 for nf4_dequantize;
 *                 the matmuls (GEMV, GEMM and their variants) take 64 only
 *                 and return NF4_ERR_UNSUPPORTED for the others
 *   dq_blocksize  256; dq_code nf4_dq_code
 *   quant_type    nf4_quant_type of the codes (0 = NF4: a zero-initialised
 *                 descriptor describes NF4 codes) */
typedef struct {
  const uint8_t *packed;
  const float *absmax;
  const uint8_t *absmax_q;
  const float *absmax_scale;
  const float *absmax_mean;
  int64_t rows, cols;
  int32_t blocksize, dq_blocksize, dq_code;
  int32_t quant_type;
} nf4_weight;

/* Blockwise NF4 quantization, [bnb-tools] "How it works" Steps 1-4.
 * For each block of `blocksize` consecutive elements (the last may be short):
 * a = max|w|; x = fp32(w / a); code = index of the nearest NF4 level (ties to
 * the lower index; every code 7 when a == 0); two codes per byte.
 *   src         device, n elements of src_dtype (NF4_F32 or NF4_BF16); 16-byte aligned
 *   packed_out  device, ceil(n/2) bytes; an odd tail's low nibble is 7 (zero code)
 *   absmax_out  device, ceil(n/blocksize) fp32 (the level-1 scales a)
 * blocksize is 32, 64, 128 or 256 (else NF4_ERR_UNSUPPORTED); 64 is the size
 * the matmuls take. */
NF4_API nf4_status nf4_quantize(const void *src, int32_t src_dtype, int64_t n, int32_t blocksize,
                        uint8_t *packed_out, float *absmax_out, nf4_stream_t stream);

/* nf4_quantize with the code book chosen by quant_type (nf4_quant_type): the
 * same blocking, absmax, packing and arguments; with NF4_QUANT_FP4 the code of
 * x = fp32(w / a) is the nearest FP4 level (see nf4_quant_type), an all-zero
 * block is all +0 codes and an odd tail's low nibble is 0.
 * nf4_quantize(...) is nf4_quantize_typed(..., NF4_QUANT_NF4, ...). */
NF4_API nf4_status nf4_quantize_typed(const void *src, int32_t src_dtype, int64_t n, int32_t blocksize,
                                      int32_t quant_type, uint8_t *packed_out, float *absmax_out,
                                      nf4_stream_t stream);

/* nf4_quantize_typed of up to NF4_QUANT_MANY_MAX tensors of one source dtype,
 * block size and code book in one launch (a model's linear layers quantized
 * as it loads, [bnb-tut] "4-bit Loading with NF4"): tensor i gets exactly the
 * packed codes and absmax that nf4_quantize_typed gives it.
 *   src, n, packed_out, absmax_out   host arrays of `count` entries: each
 *               tensor's device pointers and element count, as in nf4_quantize
 *   count       1 .. NF4_QUANT_MANY_MAX
 * A tensor with n == 0 is skipped.  Every tensor is checked before anything
 * launches; the first error is returned and nothing runs.  Tensors and
 * outputs must not overlap one another. */
#define NF4_QUANT_MANY_MAX 256
NF4_API nf4_status nf4_quantize_many(const void *const *src, const int64_t *n, int32_t count, int32_t src_dtype,
                                     int32_t blocksize, int32_t quant_type, uint8_t *const *packed_out,
                                     float *const *absmax_out, nf4_stream_t stream);

/* Double quantization of the fp32 absmax array, [bnb-tut] "How NF4 Works"
 * (scale constants quantized from float32 to float8) and [bnb-tools] "Double
 * quantization".  mu = fp32(fp64(exact sum of absmax) / nb) (one per tensor);
 * r = fp32(absmax - mu); per block of dq_blocksize: m = max|r| (stored in
 * scale_out), y = fp32(fp32(r / m) * Q), q = E4M3 round-to-nearest-even with
 * saturation (Q = 448) or int8 round-half-away clamped to +-127 (Q = 127).
 *   absmax      device, nb fp32 (finite, any sign)
 *   q_out       device, nb bytes (E4M3 bits, or int8 two's complement)
 *   scale_out   device, ceil(nb/dq_blocksize) fp32
 *   mean_out    device, 1 fp32 (4-byte aligned)
 *   workspace   device scratch of nf4_double_quant_workspace_bytes(nb) bytes,
 *               16-byte aligned, owned by the caller.  Zero-fill it before its
 *               first use; every call that completes leaves it ready for the
 *               next one (no clearing between calls).  Calls that may run at
 *               the same time need separate buffers; after
 *               nf4_check_device_error reports an error, zero it again.
 * dq_blocksize must be 256.  nb == 0 launches nothing and leaves mean_out unset.
 * Limit: nb <= NF4_DQ_MAX_NB.  The exact sum is kept as 32-bit digits in
 * signed 64-bit limbs, which stay exact for up to 2^31 - 1 values; larger nb
 * returns NF4_ERR_INVALID_ARG. */
#define NF4_DQ_MAX_NB 2147483647LL
NF4_API nf4_status nf4_double_quant(const float *absmax, int64_t nb, int32_t dq_blocksize, int32_t dq_code,
                            uint8_t *q_out, float *scale_out, float *mean_out, void *workspace,
                            size_t workspace_bytes, nf4_stream_t stream);
NF4_API size_t nf4_double_quant_workspace_bytes(int64_t nb);

/* nf4_double_quant of up to NF4_DQ_MANY_MAX absmax arrays in two launches (a
 * model's weights quantized one after another, as [bnb-tut] "4-bit Loading with
 * NF4" loads every linear layer of an 8B model), each with its own mean: array
 * i gets exactly the q, scale and mean that nf4_double_quant gives it.
 *   absmax, nb, q_out, scale_out, mean_out   host arrays of `count` entries: the
 *               device pointers and sizes of each array, as in nf4_double_quant
 *   count       1 .. NF4_DQ_MANY_MAX
 *   workspace   device scratch of nf4_double_quant_many_workspace_bytes(count)
 *               bytes, 16-byte aligned; zero-filled before its first use, left
 *               ready by every call that completes (as for nf4_double_quant)
 * An array with nb == 0 is skipped (its mean_out stays unset).  Every array is
 * checked before anything launches; the first error is returned and nothing
 * runs.  Arrays and outputs must not overlap one another. */
#define NF4_DQ_MANY_MAX 256
NF4_API nf4_status nf4_double_quant_many(const float *const *absmax, const int64_t *nb, int32_t count,
                                         int32_t dq_blocksize, int32_t dq_code, uint8_t *const *q_out,
                                         float *const *scale_out, float *const *mean_out, void *workspace,
                                         size_t workspace_bytes, nf4_stream_t stream);
NF4_API size_t nf4_double_quant_many_workspace_bytes(int32_t count);

/* nf4_double_quant without a caller-provided workspace, for callers that
 * cannot allocate device memory: code that runs under a fixed memory budget
 * set at start-up, or inside a host framework that owns the device allocator
 * and hands out no scratch.  (The pages have no counterpart to this call; it
 * only changes where the scratch lives.)
 *   Same arguments and results as nf4_double_quant, minus the workspace.  The
 *   scratch is a 256-byte static array inside the library: every GPU that
 *   loads the library holds it until the process exits.  The function itself
 *   allocates nothing (no cudaMalloc, no cudaFree).
 *   The first call on a device looks up the array's device address with that
 *   device current; make that first call before any stream capture.
 *   Every call clears the array on `stream` before using it, and all calls
 *   share it: calls that can run on the GPU at the same time (different
 *   streams, other host threads) race and must be ordered by the caller.
 *   Limit: nb <= NF4_DQ_NOALLOC_MAX_NB (the exact-sum digits in the array
 *   stay exact up to this count); larger nb returns NF4_ERR_INVALID_ARG. */
#define NF4_DQ_NOALLOC_MAX_NB NF4_DQ_MAX_NB
NF4_API nf4_status nf4_double_quant_noalloc(const float *absmax, int64_t nb, int32_t dq_blocksize, int32_t dq_code,
                                            uint8_t *q_out, float *scale_out, float *mean_out, nf4_stream_t stream);

/* Dequantization, [bnb-tools] Step 5 ("Dequantization": expand back to a higher
 * precision with the scale and the code book).  With double quantization the
 * scale is first reconstructed: a^ = fp32(fp32(fp32(dec(q)/Q) * m) + mu).
 * w^ = fp32(code[idx] * a^); out = w^ (NF4_F32) or bf16_rn(w^) (NF4_BF16).
 *   w    weight descriptor (rows*cols elements; rows/cols need no alignment;
 *        blocksize 32, 64, 128 or 256, else NF4_ERR_UNSUPPORTED)
 *   out  device, rows*cols elements of out_dtype, 16-byte aligned */
NF4_API nf4_status nf4_dequantize(const nf4_weight *w, void *out, int32_t out_dtype, nf4_stream_t stream);

/* Decode GEMV, [bnb-tools] Step 5 (expand each block to 16-bit with its scale
 * and the code book, then multiply) with bf16 compute ([bnb-tut] "4-bit
 * Loading with NF4", bnb_4bit_compute_dtype=bfloat16):
 *   y[b, n] = bf16_rn( sum_k Wc[n, k] * x[b, k] ),  Wc = bf16_rn(w^)
 * accumulated in fp32 (order unspecified).
 *   x  device bf16 [batch, cols] row-major;  y  device bf16 [batch, rows]
 *   1 <= batch <= 8; cols % 64 == 0; rows % 16 == 0. */
NF4_API nf4_status nf4_gemv(const nf4_weight *w, const void *x, int32_t batch, void *y, nf4_stream_t stream);

/* nf4_gemv for up to 4 weights that read the same input, in one launch (the
 * q/k/v projections of an attention block, or gate/up of an MLP, in the
 * decode pass over a whole 4-bit model such as the Llama-3.1-8B of [bnb-tut]
 * "4-bit Loading with NF4").  Each weight gets exactly the results nf4_gemv
 * would give it.
 *   ws     host array of `count` weight descriptors (1 <= count <= 4), all
 *          with the same cols, scale kind (plain or double-quant) and quant_type
 *   x      device bf16 [batch, cols];  ys  host array of `count` device bf16
 *          outputs, ys[i] of shape [batch, ws[i]->rows]
 *   1 <= batch <= 8; cols % 64 == 0; every rows % 16 == 0. */
NF4_API nf4_status nf4_gemv_grouped(const nf4_weight *const *ws, int32_t count, const void *x, int32_t batch,
                            void *const *ys, nf4_stream_t stream);

/* Decode GEMV over a list of weights, each with its own input and output, in
 * one launch: the decode pass over the linear layers of a whole 4-bit model
 * (such as the Llama-3.1-8B of [bnb-tut] "4-bit Loading with NF4"), each
 * block expanded on the fly as in [bnb-tools] Step 5.  Every weight gets
 * exactly the results nf4_gemv would give it:
 *   ys[i][b, n] = bf16_rn( sum_k Wc_i[n, k] * xs[i][b, k] )
 * The weights' 16-row tiles are spread over one persistent grid (one CTA per
 * SM), so small and large weights share the GPU and the pass pays one launch.
 *   ws     host array of `count` weight descriptors (by value), each with its
 *          own shape and scale kind, all with the same quant_type;
 *          rows % 16 == 0, cols % 64 == 0
 *   xs     host array of `count` device bf16 inputs, xs[i] of shape
 *          [batch, ws[i].cols], 16-byte aligned
 *   ys     host array of `count` device bf16 outputs, ys[i] of shape
 *          [batch, ws[i].rows], 4-byte aligned; no output may overlap any
 *          input or another output
 *   1 <= count <= NF4_GEMV_STREAM_MAX; 1 <= batch <= 8.
 * Weights with rows == 0 or cols == 0 are skipped. */
#define NF4_GEMV_STREAM_MAX 256
NF4_API nf4_status nf4_gemv_stream(const nf4_weight *ws, const void *const *xs, void *const *ys, int32_t count,
                                   int32_t batch, nf4_stream_t stream);

/* Prefill GEMM, same arithmetic as nf4_gemv for m activation rows:
 *   Y[m, n] = bf16_rn( sum_k Wc[n, k] * X[m, k] )
 * on tcgen05 tensor cores (bf16 x bf16 -> fp32 in tensor memory).
 *   x  device bf16 [m, cols];  y  device bf16 [m, rows];  m >= 1
 *   cols % 64 == 0; rows % 128 == 0.
 *   workspace  device scratch of nf4_gemm_workspace_bytes(w, m) bytes (may be
 *              NULL when that size is 0), 16-byte aligned, owned by the
 *              caller.  Zero-fill it before its first use; every call that
 *              completes leaves it ready for the next (no clearing between
 *              calls).  Calls that may run at the same time need separate
 *              buffers; after nf4_check_device_error reports an error, zero it
 *              again. */
NF4_API nf4_status nf4_gemm(const nf4_weight *w, const void *x, int64_t m, void *y, void *workspace,
                    size_t workspace_bytes, nf4_stream_t stream);
NF4_API size_t nf4_gemm_workspace_bytes(const nf4_weight *w, int64_t m);

/* A low-rank adapter on a frozen 4-bit weight, as QLoRA trains it ([bnb-tut]
 * "QLoRA: Fine-Tuning a 4-bit Model"; [bnb-tools] "Fine-tuning with adapters
 * on a 4-bit model": r = 16, lora_alpha = 32, scale = lora_alpha / r).
 *   down   device bf16 [r, cols] (the adapter's first map, A), 16-byte aligned
 *   up     device bf16 [rows, r] (the second map, B), 16-byte aligned
 *   r      16 or 32;  scale  finite fp32
 * nf4_gemm_lora and nf4_gemm_dx take NF4 codes only (NF4_ERR_UNSUPPORTED for
 * quant_type FP4). */
typedef struct {
  const void *down;
  const void *up;
  int32_t r;
  float scale;
} nf4_lora;

/* nf4_gemm with the adapter added in the same accumulator:
 *   v[m, j] = scale * sum_k X[m, k] * down[j, k]              (fp32 sum)
 *   Y[m, n] = bf16_rn( sum_k Wc[n, k] * X[m, k] + sum_j v[m, j] * up[n, j] )
 * v is not rounded to bf16: it reaches the tensor cores as a bf16 pair
 * (hi = bf16_rn(v), lo = bf16_rn(v - hi); about 16 significant bits).  Two
 * launches: the down map (v into the workspace), then the tcgen05 GEMM, which
 * treats [hi | lo] as one more reduction stage of each output tile with
 * [up | up] as that stage's weight.  Dropout is not applied.
 *   x  device bf16 [m, cols];  y  device bf16 [m, rows];  m >= 1
 *   cols % 64 == 0; rows % 128 == 0.
 *   workspace  device scratch of nf4_gemm_lora_workspace_bytes(w, m) bytes,
 *              16-byte aligned, never NULL for m >= 1: v, then the split
 *              scratch under nf4_gemm's contract (zero-fill before the first
 *              use, left ready by every completed call). */
NF4_API nf4_status nf4_gemm_lora(const nf4_weight *w, const nf4_lora *lora, const void *x, int64_t m, void *y,
                         void *workspace, size_t workspace_bytes, nf4_stream_t stream);
NF4_API size_t nf4_gemm_lora_workspace_bytes(const nf4_weight *w, int64_t m);

/* Input gradient of nf4_gemm, for training adapters on a frozen 4-bit base
 * ([bnb-tools] "Strengths and limitations": the quantized weights are not
 * trained, yet the loss gradient must pass through them to reach the
 * adapters; [bnb-tut] "QLoRA: Fine-Tuning a 4-bit Model": only the adapters
 * train, the 4-bit base is fixed):
 *   dX[m, k] = bf16_rn( sum_n dY[m, n] * Wc[n, k] ),  Wc as in nf4_gemv,
 * on tcgen05 tensor cores, accumulated in fp32 (order unspecified).  The
 * packed weight is read in its stored [rows, cols] layout; no transposed copy
 * is made.
 *   dy  device bf16 [m, rows] (the gradient of Y);  dx  device bf16 [m, cols]
 *   m >= 1; rows % 64 == 0; cols % 128 == 0 (else NF4_ERR_UNSUPPORTED).
 *   workspace  device scratch of nf4_gemm_dx_workspace_bytes(w, m) bytes, with
 *              the same contract as nf4_gemm's workspace (zero-fill before its
 *              first use; left ready by every completed call; separate
 *              buffers for calls that may overlap). */
NF4_API nf4_status nf4_gemm_dx(const nf4_weight *w, const void *dy, int64_t m, void *dx, void *workspace,
                       size_t workspace_bytes, nf4_stream_t stream);
NF4_API size_t nf4_gemm_dx_workspace_bytes(const nf4_weight *w, int64_t m);

/* Bytes of a quantized tensor of n elements: ceil(n/2) codes + either
 * 4*ceil(n/blocksize) (fp32 absmax) or ceil(n/blocksize) 8-bit codes +
 * 4*ceil(nb/dq_blocksize) + 4 (double quant).  Host only. */
NF4_API size_t nf4_storage_bytes(int64_t n, int32_t blocksize, int32_t double_quant, int32_t dq_blocksize);

/* Synchronizes `stream`, then reports and clears the device error word of the
 * current device: NF4_OK, or NF4_ERR_TIMEOUT if a device-side bounded wait
 * gave up since the last check; NF4_ERR_CUDA if the stream reports an error. */
NF4_API nf4_status nf4_check_device_error(nf4_stream_t stream);

/* Static string naming a status. Host only. */
NF4_API const char *nf4_status_string(nf4_status s);

/* The library's 16 NF4 levels (ascending, index 7 = 0.0f), copied to host
 * memory `out`.  Host only. */
NF4_API void nf4_code_table(float out[16]);

/* 1 if the current CUDA device is sm_100 (B200 class), else 0. */
NF4_API int32_t nf4_device_supported(void);

/* Diagnostics: number of kernels this process has launched through the
 * library so far (all devices, all threads).  Host only. */
NF4_API uint64_t nf4_kernel_launches(void);

/* Self-test of the failure path shared by every bounded device-side wait:
 * launches one CTA that waits on an mbarrier nothing completes.  After the
 * library's wall-clock bound (2 s) the wait gives up, records a timeout in the
 * device error word and the kernel returns, so the context stays usable; the
 * next nf4_check_device_error(stream) reports NF4_ERR_TIMEOUT (and clears it).
 * Returns the launch status. */
NF4_API nf4_status nf4_selftest_wait_timeout(nf4_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* NF4_H */
