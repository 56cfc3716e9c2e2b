/*
 * nf4_oracle.c -- plain, slow, obviously correct CPU oracle (TEST INFRASTRUCTURE).
 *
 * Only tests, the package smoke check and the benchmark's CPU-baseline leg may
 * call this file.  It is compiled with -O2 -ffp-contract=off -fno-fast-math so
 * every float operation below is one IEEE-754 operation rounded to nearest even
 * in the precision of its operands.  Loops marked "parallel" only distribute
 * independent outputs over threads; they do not reorder any arithmetic.
 *
 * Page citations:
 *   [bnb-tools] "bitsandbytes" (ozercemkelahmet.com/tools/bitsandbytes)
 *   [bnb-tut]   "bitsandbytes quantization tutorial: 4-bit and 8-bit models" (mljourney.com)
 */
#include "nf4_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int g_threads = 0;

void oracle_set_threads(int n) {
  g_threads = n;
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#endif
}

int oracle_get_threads(void) {
#ifdef _OPENMP
  return g_threads > 0 ? g_threads : omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------------- */
/* NF4 code book.                                                             */
/*                                                                            */
/* [bnb-tools] "How NF4 works": the 16 levels split the normal distribution  */
/* of the weights into pieces of equal probability.                          */
/* [bnb-tut] "How NF4 Works": a grid for normally distributed data, levels    */
/* densest near zero.  The QLoRA construction read here: quantiles of N(0,1)  */
/* taken at equally spaced probabilities, 8 on the positive side and 7 on the */
/* negative side of an exact zero, scaled so the extremes are -1 and +1.  The */
/* outermost probability p* is the average of the half-bin ends for 30 and 32 */
/* bins, which keeps the extreme quantile finite.                             */
/* ------------------------------------------------------------------------- */

/* standard normal CDF */
static double phi(double z) { return 0.5 * erfc(-z / sqrt(2.0)); }

/* inverse of phi by bisection: phi is increasing, so keep [lo, hi] bracketing p */
static double phi_inv(double p) {
  double lo = -40.0, hi = 40.0;
  for (int it = 0; it < 400; ++it) {
    double mid = 0.5 * (lo + hi);
    if (mid == lo || mid == hi) break;
    if (phi(mid) < p) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

void oracle_nf4_codebook(double c64[16], float c32[16]) {
  const double pstar = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
  double v[16];
  int m = 0;
  /* negative side: 7 of 8 equally spaced probabilities in [0.5, p*], excluding 0.5 */
  for (int k = 7; k >= 1; --k) v[m++] = -phi_inv(0.5 + (pstar - 0.5) * ((double)k / 7.0));
  v[m++] = 0.0;
  /* positive side: 8 of 9 equally spaced probabilities in [0.5, p*], excluding 0.5 */
  for (int k = 1; k <= 8; ++k) v[m++] = phi_inv(0.5 + (pstar - 0.5) * ((double)k / 8.0));
  double vmax = 0.0;
  for (int i = 0; i < 16; ++i) vmax = fabs(v[i]) > vmax ? fabs(v[i]) : vmax;
  for (int i = 0; i < 16; ++i) {
    c64[i] = v[i] / vmax;
    c32[i] = (float)c64[i];
  }
}

static float g_code[16];
static int g_code_ready = 0;

static const float *codebook32(void) {
  if (!g_code_ready) {
    double c64[16];
    float c32[16];
    oracle_nf4_codebook(c64, c32);
    memcpy(g_code, c32, sizeof c32);
    g_code_ready = 1;
  }
  return g_code;
}

/* ------------------------------------------------------------------------- */
/* bf16 <-> fp32                                                              */
/* ------------------------------------------------------------------------- */

uint16_t oracle_bf16_rn(float v) {
  uint32_t u;
  memcpy(&u, &v, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u); /* NaN stays NaN */
  uint32_t keep_lsb = (u >> 16) & 1u;
  u += 0x7fffu + keep_lsb; /* add half an ulp (minus one on an even tie) then truncate */
  return (uint16_t)(u >> 16);
}

float oracle_bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* ------------------------------------------------------------------------- */
/* Level-1 quantization: [bnb-tools] "How it works" Steps 1-4.                */
/* ------------------------------------------------------------------------- */

/* Step 3: the nearest entry of the code book.  Distances are exact in fp64
 * (difference of two fp32 numbers); a tie keeps the lower index. */
int oracle_nf4_nearest_code(float x) {
  const float *c = codebook32();
  int best = 0;
  double bd = fabs((double)x - (double)c[0]);
  for (int i = 1; i < 16; ++i) {
    double d = fabs((double)x - (double)c[i]);
    if (d < bd) { bd = d; best = i; }
  }
  return best;
}

void oracle_nf4_quantize_f32(const float *w, int64_t n, int32_t blocksize,
                             uint8_t *packed, float *absmax) {
  int64_t nb = (n + blocksize - 1) / blocksize;
  uint8_t *idx = (uint8_t *)malloc((size_t)(n > 0 ? n : 1));
  (void)codebook32(); /* derive the table before the threads read it */
  /* Step 1: blocks of `blocksize` consecutive values (the last may be short) */
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < nb; ++b) {
    int64_t lo = b * blocksize, hi = lo + blocksize < n ? lo + blocksize : n;
    /* Step 2: the block's largest absolute value is its scale */
    float a = 0.0f;
    for (int64_t i = lo; i < hi; ++i) a = fabsf(w[i]) > a ? fabsf(w[i]) : a;
    absmax[b] = a;
    for (int64_t i = lo; i < hi; ++i) {
      if (a == 0.0f) { idx[i] = 7; continue; } /* all-zero block: every value is the zero code */
      float x = w[i] / a;                       /* Step 2: divide by it -> [-1, 1] (fp32) */
      idx[i] = (uint8_t)oracle_nf4_nearest_code(x); /* Step 3 */
    }
  }
  /* Step 4: two values share one byte; the even element takes the high nibble,
   * an odd tail's missing partner is the zero code */
  for (int64_t j = 0; j < (n + 1) / 2; ++j) {
    uint8_t hi4 = idx[2 * j];
    uint8_t lo4 = (2 * j + 1 < n) ? idx[2 * j + 1] : 7;
    packed[j] = (uint8_t)((hi4 << 4) | lo4);
  }
  free(idx);
}

void oracle_nf4_quantize_bf16(const uint16_t *w, int64_t n, int32_t blocksize,
                              uint8_t *packed, float *absmax) {
  float *wf = (float *)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
  for (int64_t i = 0; i < n; ++i) wf[i] = oracle_bf16_to_f32(w[i]); /* exact widening */
  oracle_nf4_quantize_f32(wf, n, blocksize, packed, absmax);
  free(wf);
}

/* ------------------------------------------------------------------------- */
/* Exact sum.  Every finite fp32 value is an integer multiple of 2^-149, so    */
/* the sum is an integer times 2^-149; it is kept as a 384-bit integer in     */
/* 32-bit limbs (positive and negative parts apart) and rounded once to fp64. */
/* ------------------------------------------------------------------------- */

#define NLIMB 12

static void big_add(uint64_t *limb, uint32_t mant, int shift) {
  /* limb[] += mant * 2^shift; limbs hold 32 significant bits each, and the
   * spare upper 32 bits absorb carries until normalisation */
  int li = shift / 32, s = shift % 32;
  uint64_t v = (uint64_t)mant << s; /* at most 24 + 31 bits */
  limb[li] += v & 0xffffffffu;
  limb[li + 1] += v >> 32;
}

static void big_normalise(uint64_t *limb) {
  for (int i = 0; i < NLIMB - 1; ++i) {
    limb[i + 1] += limb[i] >> 32;
    limb[i] &= 0xffffffffu;
  }
}

/* a >= b assumed, both normalised: a -= b */
static void big_sub(uint64_t *a, const uint64_t *b) {
  int64_t borrow = 0;
  for (int i = 0; i < NLIMB; ++i) {
    int64_t d = (int64_t)a[i] - (int64_t)b[i] - borrow;
    borrow = d < 0;
    a[i] = (uint64_t)(d + (borrow ? ((int64_t)1 << 32) : 0));
  }
}

static int big_cmp(const uint64_t *a, const uint64_t *b) {
  for (int i = NLIMB - 1; i >= 0; --i)
    if (a[i] != b[i]) return a[i] > b[i] ? 1 : -1;
  return 0;
}

static int big_bit(const uint64_t *x, int k) { return (int)((x[k / 32] >> (k % 32)) & 1u); }

/* value of the normalised integer x times 2^-149, rounded to nearest even fp64 */
static double big_to_double(const uint64_t *x) {
  int top = -1;
  for (int k = NLIMB * 32 - 1; k >= 0; --k)
    if (big_bit(x, k)) { top = k; break; }
  if (top < 0) return 0.0;
  if (top < 53) {
    uint64_t m = 0;
    for (int k = top; k >= 0; --k) m = (m << 1) | (uint64_t)big_bit(x, k);
    return ldexp((double)m, -149);
  }
  uint64_t m = 0;
  for (int k = top; k >= top - 52; --k) m = (m << 1) | (uint64_t)big_bit(x, k);
  int round = big_bit(x, top - 53);
  int sticky = 0;
  for (int k = top - 54; k >= 0 && !sticky; --k) sticky = big_bit(x, k);
  if (round && (sticky || (m & 1u))) m += 1; /* may reach 2^53: still exact in fp64 */
  return ldexp((double)m, top - 52 - 149);
}

double oracle_exact_sum_f32(const float *a, int64_t n) {
  uint64_t pos[NLIMB], neg[NLIMB];
  memset(pos, 0, sizeof pos);
  memset(neg, 0, sizeof neg);
  for (int64_t i = 0; i < n; ++i) {
    uint32_t u;
    memcpy(&u, &a[i], 4);
    uint32_t e = (u >> 23) & 0xffu, f = u & 0x7fffffu;
    /* normal: (2^23 + f) * 2^(e-150) = (2^23+f)*2^(e-1) * 2^-149;
     * subnormal: f * 2^-149 (same formula with e = 1 and no hidden bit) */
    uint32_t mant = e ? (f | 0x800000u) : f;
    int shift = e ? (int)e - 1 : 0;
    big_add((u >> 31) ? neg : pos, mant, shift);
    if ((i & 0xffffff) == 0xffffff) { big_normalise(pos); big_normalise(neg); }
  }
  big_normalise(pos);
  big_normalise(neg);
  if (big_cmp(pos, neg) >= 0) {
    big_sub(pos, neg);
    return big_to_double(pos);
  }
  big_sub(neg, pos);
  return -big_to_double(neg);
}

/* ------------------------------------------------------------------------- */
/* OCP FP8 E4M3 ("float8" in [bnb-tut] "How NF4 Works": the per-block scale  */
/* constants are quantised from float32 to float8).  Bit layout s.eeee.mmm,  */
/* exponent bias 7, subnormals m*2^-9, no infinities, s.1111.111 is NaN.      */
/* ------------------------------------------------------------------------- */

float oracle_e4m3_decode(uint8_t code) {
  int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  double mag = e == 0 ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
  return (float)(s ? -mag : mag);
}

/* nearest finite E4M3 value (ties to the even code), magnitudes >= 448 clamp */
uint8_t oracle_e4m3_encode_satfinite(float y) {
  uint32_t u;
  memcpy(&u, &y, 4);
  uint8_t sign = (uint8_t)((u >> 31) << 7);
  double ay = fabs((double)y);
  if (ay >= 448.0) return (uint8_t)(sign | 0x7e);
  int best = 0;
  double bd = ay; /* distance to code 0 (+0) */
  for (int c = 1; c <= 0x7e; ++c) {
    double d = fabs(ay - (double)oracle_e4m3_decode((uint8_t)c));
    if (d < bd || (d == bd && (c & 1) == 0)) { bd = d; best = c; }
  }
  return (uint8_t)(sign | best);
}

/* ------------------------------------------------------------------------- */
/* Second-level (8-bit) blockwise quantization.                               */
/* [bnb-tools] "Double quantization": the per-block scales are themselves     */
/* quantized.  The recipe follows [bnb-tools] "A worked example": take the    */
/* block absmax, divide by it, multiply by the top code (127 for int8; 448,   */
/* the largest E4M3 value, for float8) and round; to dequantize, divide by    */
/* the top code and multiply by the absmax.  int8 rounding is half away from  */
/* zero as in that example; float8 is round-to-nearest-even onto the E4M3     */
/* grid, saturating at +-448.                                                 */
/* ------------------------------------------------------------------------- */

static float dq_top(int code) { return code == ORACLE_DQ_E4M3 ? 448.0f : 127.0f; }

static float dq_decode(uint8_t q, int code) {
  return code == ORACLE_DQ_E4M3 ? oracle_e4m3_decode(q) : (float)(int8_t)q;
}

void oracle_blockwise_8bit(const float *v, int64_t n, int32_t blocksize, int code,
                           uint8_t *q, float *scale) {
  const float Q = dq_top(code);
  int64_t ng = (n + blocksize - 1) / blocksize;
  for (int64_t g = 0; g < ng; ++g) {
    int64_t lo = g * blocksize, hi = lo + blocksize < n ? lo + blocksize : n;
    float m = 0.0f;
    for (int64_t j = lo; j < hi; ++j) m = fabsf(v[j]) > m ? fabsf(v[j]) : m;
    scale[g] = m;
    for (int64_t j = lo; j < hi; ++j) {
      float y = 0.0f;
      if (m != 0.0f) {
        float x = v[j] / m; /* into [-1, 1] */
        y = x * Q;          /* onto the code's range */
      }
      if (code == ORACLE_DQ_E4M3) {
        q[j] = oracle_e4m3_encode_satfinite(y);
      } else {
        float t = roundf(y); /* half away from zero */
        if (t > 127.0f) t = 127.0f;
        if (t < -127.0f) t = -127.0f;
        q[j] = (uint8_t)(int8_t)t;
      }
    }
  }
}

float oracle_blockwise_8bit_value(uint8_t q, float scale, int code) {
  float unit = dq_decode(q, code) / dq_top(code); /* back to [-1, 1] */
  return unit * scale;
}

/* Double quantization of the absmax array.  The mean is one fp32 scalar per
 * tensor: the exact sum rounded to fp64, divided by the count in fp64, rounded
 * to fp32.  Residuals are taken in fp32. */
void oracle_nf4_double_quant(const float *absmax, int64_t nb, int32_t dq_blocksize, int code,
                             uint8_t *q, float *scale, float *mean) {
  if (nb <= 0) { *mean = 0.0f; return; }
  double s = oracle_exact_sum_f32(absmax, nb);
  float mu = (float)(s / (double)nb);
  float *r = (float *)malloc((size_t)nb * sizeof(float));
  for (int64_t j = 0; j < nb; ++j) r[j] = absmax[j] - mu;
  oracle_blockwise_8bit(r, nb, dq_blocksize, code, q, scale);
  free(r);
  *mean = mu;
}

void oracle_absmax_reconstruct(const uint8_t *q, const float *scale, float mean, int64_t nb,
                               int32_t dq_blocksize, int code, float *out) {
  for (int64_t j = 0; j < nb; ++j)
    out[j] = oracle_blockwise_8bit_value(q[j], scale[j / dq_blocksize], code) + mean;
}

/* ------------------------------------------------------------------------- */
/* Dequantization: [bnb-tools] Step 5 -- read a block, expand it with the     */
/* scale and the code book: w^ = c[idx] * a in fp32.                          */
/* ------------------------------------------------------------------------- */

static int code_at(const uint8_t *packed, int64_t i) {
  uint8_t byte = packed[i / 2];
  return (i % 2 == 0) ? (byte >> 4) : (byte & 15);
}

void oracle_nf4_dequantize_f32(const uint8_t *packed, const float *absmax, int64_t n,
                               int32_t blocksize, float *out) {
  const float *c = codebook32();
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = c[code_at(packed, i)] * absmax[i / blocksize];
}

void oracle_nf4_dequantize_bf16(const uint8_t *packed, const float *absmax, int64_t n,
                                int32_t blocksize, uint16_t *out) {
  const float *c = codebook32();
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = oracle_bf16_rn(c[code_at(packed, i)] * absmax[i / blocksize]);
}

/* ------------------------------------------------------------------------- */
/* Matmul with on-the-fly dequantization.  [bnb-tools] Step 5: the block is   */
/* expanded back to 16-bit with the scale and code book, then multiplied;     */
/* [bnb-tut] "4-bit Loading with NF4": compute dtype bfloat16.  The expanded  */
/* weight is Wc = bf16_rn(c[idx] * a); products of two bf16 values are exact  */
/* in fp64 and are summed in fp64.                                            */
/* ------------------------------------------------------------------------- */

static double dot_row_cb(const uint8_t *packed, const float *absmax, int64_t K, int32_t blocksize,
                         int64_t n, const uint16_t *xrow, const float *c) {
  double acc = 0.0;
  for (int64_t k = 0; k < K; ++k) {
    int64_t i = n * K + k;
    float wc = oracle_bf16_to_f32(oracle_bf16_rn(c[code_at(packed, i)] * absmax[i / blocksize]));
    acc += (double)wc * (double)oracle_bf16_to_f32(xrow[k]);
  }
  return acc;
}

static double dot_row(const uint8_t *packed, const float *absmax, int64_t K, int32_t blocksize,
                      int64_t n, const uint16_t *xrow) {
  return dot_row_cb(packed, absmax, K, blocksize, n, xrow, codebook32());
}

void oracle_nf4_matmul(const uint8_t *packed, const float *absmax, int64_t N, int64_t K,
                       int32_t blocksize, const uint16_t *x, int64_t B, double *y) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t b = 0; b < B; ++b) y[b * N + n] = dot_row(packed, absmax, K, blocksize, n, x + b * K);
}

void oracle_nf4_matmul_sampled(const uint8_t *packed, const float *absmax, int64_t N, int64_t K,
                               int32_t blocksize, const uint16_t *x, int64_t B,
                               const int64_t *bs, const int64_t *ns, int64_t count, double *y) {
  (void)N;
  (void)B;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < count; ++t) y[t] = dot_row(packed, absmax, K, blocksize, ns[t], x + bs[t] * K);
}

/* ------------------------------------------------------------------------- */
/* Input gradient of the same matmul.  [bnb-tools] "Strengths and            */
/* limitations" (Limitations) and [bnb-tut] "QLoRA: Fine-Tuning a 4-bit       */
/* Model": the 4-bit base weight is not trained (it gets no gradient of its  */
/* own), yet the loss gradient has to pass through it to reach the adapters  */
/* and the layers below:                                                      */
/* dx[b,k] = sum_n dy[b,n] * Wc[n,k], with Wc the same 16-bit expanded weight */
/* as above.  Products of two bf16 values are exact in fp64; summed in fp64   */
/* over n in ascending order.                                                 */
/* ------------------------------------------------------------------------- */

static double dot_col(const uint8_t *packed, const float *absmax, int64_t N, int64_t K,
                      int32_t blocksize, int64_t k, const uint16_t *dyrow) {
  const float *c = codebook32();
  double acc = 0.0;
  for (int64_t n = 0; n < N; ++n) {
    int64_t i = n * K + k;
    float wc = oracle_bf16_to_f32(oracle_bf16_rn(c[code_at(packed, i)] * absmax[i / blocksize]));
    acc += (double)oracle_bf16_to_f32(dyrow[n]) * (double)wc;
  }
  return acc;
}

void oracle_nf4_matmul_dx(const uint8_t *packed, const float *absmax, int64_t N, int64_t K,
                          int32_t blocksize, const uint16_t *dy, int64_t B, double *dx) {
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < K; ++k)
    for (int64_t b = 0; b < B; ++b) dx[b * K + k] = dot_col(packed, absmax, N, K, blocksize, k, dy + b * N);
}

void oracle_nf4_matmul_dx_sampled(const uint8_t *packed, const float *absmax, int64_t N, int64_t K,
                                  int32_t blocksize, const uint16_t *dy, int64_t B,
                                  const int64_t *bs, const int64_t *ks, int64_t count, double *dx) {
  (void)B;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < count; ++t) dx[t] = dot_col(packed, absmax, N, K, blocksize, ks[t], dy + bs[t] * N);
}

/* ------------------------------------------------------------------------- */
/* The 4-bit matmul with a low-rank adapter added, as QLoRA trains it:        */
/* [bnb-tut] "QLoRA: Fine-Tuning a 4-bit Model" and [bnb-tools] "Fine-tuning  */
/* with adapters on a 4-bit model" (LoraConfig r = 16, lora_alpha = 32: the   */
/* frozen 4-bit base plus small trainable adapter matrices).  The adapter is  */
/* the usual pair of bf16 linear maps, down A [r, K] and up B [N, r], scaled  */
/* by s = lora_alpha / r, with no rounding of the intermediate:               */
/*   t[b,j]  = s * sum_k x[b,k] * A[j,k]                                       */
/*   y[b,n]  = sum_k Wc[n,k] * x[b,k] + sum_j t[b,j] * B[n,j]                  */
/* all in fp64 (products of bf16 values are exact); dropout is not part of    */
/* the product.                                                               */
/* ------------------------------------------------------------------------- */

void oracle_lora_down(const uint16_t *x, int64_t Bn, int64_t K, const uint16_t *A, int32_t r, float scale,
                      double *t) {
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < Bn; ++b)
    for (int32_t j = 0; j < r; ++j) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k)
        acc += (double)oracle_bf16_to_f32(x[b * K + k]) * (double)oracle_bf16_to_f32(A[(int64_t)j * K + k]);
      t[b * r + j] = (double)scale * acc;
    }
}

static double lora_term(const double *trow, const uint16_t *Bup, int64_t n, int32_t r) {
  double acc = 0.0;
  for (int32_t j = 0; j < r; ++j) acc += trow[j] * (double)oracle_bf16_to_f32(Bup[n * r + j]);
  return acc;
}

void oracle_nf4_matmul_lora(const uint8_t *packed, const float *absmax, int64_t N, int64_t K, int32_t blocksize,
                            const uint16_t *x, int64_t Bn, const uint16_t *A, const uint16_t *Bup, int32_t r,
                            float scale, double *y) {
  double *t = (double *)malloc(sizeof(double) * (size_t)(Bn * r > 0 ? Bn * r : 1));
  oracle_lora_down(x, Bn, K, A, r, scale, t);
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t b = 0; b < Bn; ++b)
      y[b * N + n] = dot_row(packed, absmax, K, blocksize, n, x + b * K) + lora_term(t + b * r, Bup, n, r);
  free(t);
}

/* Same arithmetic for a list of (b, n) output coordinates only (t from oracle_lora_down). */
void oracle_nf4_matmul_lora_sampled(const uint8_t *packed, const float *absmax, int64_t N, int64_t K,
                                    int32_t blocksize, const uint16_t *x, const double *t, const uint16_t *Bup,
                                    int32_t r, const int64_t *bs, const int64_t *ns, int64_t count, double *y) {
  (void)N;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i)
    y[i] = dot_row(packed, absmax, K, blocksize, ns[i], x + bs[i] * K) + lora_term(t + bs[i] * r, Bup, ns[i], r);
}

/* ------------------------------------------------------------------------- */
/* FP4 variant of the 4-bit code: [bnb-tools] "Glossary" (the FP4 entry) and */
/* "What it is" (4-bit linear layers in either format); [env-tf]             */
/* "Description".  The pages name the type but give no layout.  Reading: the */
/* OCP E2M1 format (sign, 2 exponent bits with bias 1, 1 mantissa bit, no     */
/* infinities or NaN), magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6, divided by 6 so */
/* that the block absmax maps to +-1 as with NF4.  The stored 4-bit value is  */
/* the E2M1 bit pattern s e1 e0 m itself.  Blocking, absmax, packing and      */
/* double quantization are those of NF4.                                      */
/* ------------------------------------------------------------------------- */

void oracle_fp4_codebook(double *c64, float *c32) {
  for (int nib = 0; nib < 16; ++nib) {
    int s = nib >> 3, e = (nib >> 1) & 3, m = nib & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1); /* subnormal when e == 0 */
    double v = (s ? -mag : mag) / 6.0;
    c64[nib] = v;
    c32[nib] = (float)v;
  }
}

static float g_fp4[16];
static int g_fp4_ready = 0;

static const float *fp4_codebook32(void) {
  if (!g_fp4_ready) {
    double c64[16];
    oracle_fp4_codebook(c64, g_fp4);
    g_fp4_ready = 1;
  }
  return g_fp4;
}

/* Nearest FP4 level of x (the fp32 levels, distance in exact arithmetic); a tie
 * goes to the level with an even mantissa bit (the format's round-half-even);
 * a result of zero keeps the sign of x (-0 is pattern 8). */
int oracle_fp4_nearest_code(float x) {
  const float *c = fp4_codebook32();
  int neg = signbit(x) ? 1 : 0;
  double ax = fabs((double)x);
  int best = 0; /* magnitude pattern 0..7 (levels c[0..7] ascend) */
  double bd = ax - (double)c[0];
  for (int k = 1; k < 8; ++k) {
    double d = fabs(ax - (double)c[k]);
    if (d < bd || (d == bd && (k & 1) == 0)) { bd = d; best = k; }
  }
  return (neg << 3) | best;
}

void oracle_fp4_quantize_f32(const float *w, int64_t n, int32_t blocksize, uint8_t *packed, float *absmax) {
  int64_t nb = (n + blocksize - 1) / blocksize;
  uint8_t *idx = (uint8_t *)malloc((size_t)(n > 0 ? n : 1));
  (void)fp4_codebook32();
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < nb; ++b) {
    int64_t lo = b * blocksize, hi = lo + blocksize < n ? lo + blocksize : n;
    float a = 0.0f;
    for (int64_t i = lo; i < hi; ++i) a = fabsf(w[i]) > a ? fabsf(w[i]) : a;
    absmax[b] = a;
    for (int64_t i = lo; i < hi; ++i) {
      if (a == 0.0f) { idx[i] = 0; continue; } /* all-zero block: every value is +0 */
      idx[i] = (uint8_t)oracle_fp4_nearest_code(w[i] / a);
    }
  }
  for (int64_t j = 0; j < (n + 1) / 2; ++j) {
    uint8_t hi4 = idx[2 * j];
    uint8_t lo4 = (2 * j + 1 < n) ? idx[2 * j + 1] : 0; /* an odd tail's partner is +0 */
    packed[j] = (uint8_t)((hi4 << 4) | lo4);
  }
  free(idx);
}

void oracle_fp4_quantize_bf16(const uint16_t *w, int64_t n, int32_t blocksize, uint8_t *packed, float *absmax) {
  float *wf = (float *)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
  for (int64_t i = 0; i < n; ++i) wf[i] = oracle_bf16_to_f32(w[i]);
  oracle_fp4_quantize_f32(wf, n, blocksize, packed, absmax);
  free(wf);
}

void oracle_fp4_dequantize_f32(const uint8_t *packed, const float *absmax, int64_t n, int32_t blocksize, float *out) {
  const float *c = fp4_codebook32();
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = c[code_at(packed, i)] * absmax[i / blocksize];
}

void oracle_fp4_dequantize_bf16(const uint8_t *packed, const float *absmax, int64_t n, int32_t blocksize,
                                uint16_t *out) {
  const float *c = fp4_codebook32();
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_rn(c[code_at(packed, i)] * absmax[i / blocksize]);
}

/* The 4-bit matmul of FP4 weights: the same arithmetic as oracle_nf4_matmul with
 * the FP4 levels, Wc = bf16_rn(fp4[code] * a). */
void oracle_fp4_matmul(const uint8_t *packed, const float *absmax, int64_t N, int64_t K, int32_t blocksize,
                       const uint16_t *x, int64_t B, double *y) {
  const float *c = fp4_codebook32();
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t b = 0; b < B; ++b) y[b * N + n] = dot_row_cb(packed, absmax, K, blocksize, n, x + b * K, c);
}
