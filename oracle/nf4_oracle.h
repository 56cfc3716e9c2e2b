/*
 * nf4_oracle.h -- plain CPU oracle for blockwise NF4 quantization with double
 * quantization, dequantization and the 4-bit-weight x bf16 matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this code; only the tests, the package's smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or constant generator
 * with the CUDA library: the NF4 code book is derived here from its definition.
 *
 * Sources (web pages on bitsandbytes / QLoRA):
 *   [bnb-tools]  "bitsandbytes" (ozercemkelahmet.com/tools/bitsandbytes):
 *                "How it works" Steps 1-5, "How NF4 works", "Double quantization",
 *                "A worked example", "Memory arithmetic".
 *   [bnb-tut]    "bitsandbytes quantization tutorial: 4-bit and 8-bit models"
 *                (mljourney.com): "4-bit Loading with NF4", "How NF4 Works".
 *
 * Every floating-point step is written as an explicit IEEE operation in the
 * precision stated beside it; the file is compiled with -ffp-contract=off so no
 * multiply-add is fused.  Integers fixed by the method (codes, packed bytes)
 * are therefore reproducible bit for bit.
 */
#ifndef NF4_ORACLE_H
#define NF4_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The 16 NF4 levels, ascending: fp64 before and fp32 after the final rounding. */
void oracle_nf4_codebook(double c64[16], float c32[16]);

/* Round an fp32 value to bf16 (round to nearest, ties to even); finite inputs. */
uint16_t oracle_bf16_rn(float v);
float oracle_bf16_to_f32(uint16_t b);

/* Level-1 quantization (Steps 1-4): blocks of `blocksize` consecutive values,
 * absmax scale, nearest code, two codes per byte (even element -> high nibble).
 * packed: ceil(n/2) bytes; absmax: ceil(n/blocksize) floats. */
void oracle_nf4_quantize_f32(const float *w, int64_t n, int32_t blocksize,
                             uint8_t *packed, float *absmax);
void oracle_nf4_quantize_bf16(const uint16_t *w, int64_t n, int32_t blocksize,
                              uint8_t *packed, float *absmax);

/* Nearest NF4 code index of one normalised value x (ties -> lower index). */
int oracle_nf4_nearest_code(float x);

/* Exact sum of n fp32 values, rounded once to fp64 (round to nearest even). */
double oracle_exact_sum_f32(const float *a, int64_t n);

/* OCP FP8 E4M3 ("fn": no infinities, 0x7f/0xff NaN, max finite 448). */
float oracle_e4m3_decode(uint8_t code);
uint8_t oracle_e4m3_encode_satfinite(float y);   /* nearest, ties to even, clamp */

/* 8-bit codes: 0 = E4M3 float8 (Q = 448), 1 = linear int8 (Q = 127). */
enum { ORACLE_DQ_E4M3 = 0, ORACLE_DQ_INT8 = 1 };

/* Second-level blockwise 8-bit quantization of an fp32 array with no mean
 * removal: per block the absmax m is the stored scale, x = v/m, y = x*Q, code =
 * round(y).  This is the level-1 recipe with an 8-bit code book. */
void oracle_blockwise_8bit(const float *v, int64_t n, int32_t blocksize, int code,
                           uint8_t *q, float *scale);
/* value of one 8-bit code: RN(RN(dec(q)/Q) * scale) */
float oracle_blockwise_8bit_value(uint8_t q, float scale, int code);

/* Double quantization of the level-1 absmax array: mean mu (one per tensor),
 * residuals r = a - mu, then the blockwise 8-bit recipe on r. */
void oracle_nf4_double_quant(const float *absmax, int64_t nb, int32_t dq_blocksize, int code,
                             uint8_t *q, float *scale, float *mean);
/* Reconstructed absmax a^ = RN(value(q) + mu), one per level-1 block. */
void oracle_absmax_reconstruct(const uint8_t *q, const float *scale, float mean, int64_t nb,
                               int32_t dq_blocksize, int code, float *out);

/* Dequantization (Step 5): w^ = RN(c[idx] * a).  `absmax` holds one scale per
 * block (already reconstructed when double quantization was used). */
void oracle_nf4_dequantize_f32(const uint8_t *packed, const float *absmax, int64_t n,
                               int32_t blocksize, float *out);
void oracle_nf4_dequantize_bf16(const uint8_t *packed, const float *absmax, int64_t n,
                                int32_t blocksize, uint16_t *out);

/* Matmul with on-the-fly dequantization: W is [N,K] row-major (flattened for
 * quantization), x is bf16 [B,K].  y[b,n] = sum_k Wc[n,k]*x[b,k] accumulated in
 * fp64, with Wc = bf16_rn(w^) the 16-bit expanded weight. */
void oracle_nf4_matmul(const uint8_t *packed, const float *absmax, int64_t N, int64_t K,
                       int32_t blocksize, const uint16_t *x, int64_t B, double *y);
/* Same arithmetic for a list of (b, n) output coordinates only. */
void oracle_nf4_matmul_sampled(const uint8_t *packed, const float *absmax, int64_t N, int64_t K,
                               int32_t blocksize, const uint16_t *x, int64_t B,
                               const int64_t *bs, const int64_t *ns, int64_t count, double *y);

/* Input gradient of that matmul (the frozen weight passes the loss gradient
 * to the layers below): dy is bf16 [B,N]; dx[b,k] = sum_n dy[b,n]*Wc[n,k]
 * accumulated in fp64 over n in ascending order. */
void oracle_nf4_matmul_dx(const uint8_t *packed, const float *absmax, int64_t N, int64_t K,
                          int32_t blocksize, const uint16_t *dy, int64_t B, double *dx);
/* Same arithmetic for a list of (b, k) output coordinates only. */
void oracle_nf4_matmul_dx_sampled(const uint8_t *packed, const float *absmax, int64_t N, int64_t K,
                                  int32_t blocksize, const uint16_t *dy, int64_t B,
                                  const int64_t *bs, const int64_t *ks, int64_t count, double *dx);

/* Low-rank adapter on the 4-bit matmul (QLoRA): down map A bf16 [r,K], up map
 * Bup bf16 [N,r], scale s.  t = s * x . A^T in fp64 ([Bn, r], not rounded);
 * y[b,n] = sum_k Wc[n,k]*x[b,k] + sum_j t[b,j]*Bup[n,j] in fp64. */
void oracle_lora_down(const uint16_t *x, int64_t Bn, int64_t K, const uint16_t *A, int32_t r, float scale,
                      double *t);
void oracle_nf4_matmul_lora(const uint8_t *packed, const float *absmax, int64_t N, int64_t K, int32_t blocksize,
                            const uint16_t *x, int64_t Bn, const uint16_t *A, const uint16_t *Bup, int32_t r,
                            float scale, double *y);
/* The adapter product at a list of (b, n) coordinates, given t = oracle_lora_down(x). */
void oracle_nf4_matmul_lora_sampled(const uint8_t *packed, const float *absmax, int64_t N, int64_t K,
                                    int32_t blocksize, const uint16_t *x, const double *t, const uint16_t *Bup,
                                    int32_t r, const int64_t *bs, const int64_t *ns, int64_t count, double *y);

/* FP4 (OCP E2M1 values / 6, indexed by the 4-bit pattern s e1 e0 m): code
 * book, nearest code (ties to an even mantissa bit, zero keeps the sign of x),
 * blockwise quantization (all-zero block and odd-tail partner: +0) and
 * dequantization; blocking, absmax and packing as for NF4. */
void oracle_fp4_codebook(double *c64, float *c32);
int oracle_fp4_nearest_code(float x);
void oracle_fp4_quantize_f32(const float *w, int64_t n, int32_t blocksize, uint8_t *packed, float *absmax);
void oracle_fp4_quantize_bf16(const uint16_t *w, int64_t n, int32_t blocksize, uint8_t *packed, float *absmax);
void oracle_fp4_dequantize_f32(const uint8_t *packed, const float *absmax, int64_t n, int32_t blocksize, float *out);
void oracle_fp4_dequantize_bf16(const uint8_t *packed, const float *absmax, int64_t n, int32_t blocksize,
                                uint16_t *out);

/* The 4-bit matmul with FP4 levels: y[b,n] = sum_k bf16_rn(fp4[code]*a)*x[b,k] (fp64). */
void oracle_fp4_matmul(const uint8_t *packed, const float *absmax, int64_t N, int64_t K, int32_t blocksize,
                       const uint16_t *x, int64_t B, double *y);

/* Worker threads used by the loops marked parallel (0 = OpenMP default). */
void oracle_set_threads(int n);
int oracle_get_threads(void);

#ifdef __cplusplus
}
#endif
#endif
