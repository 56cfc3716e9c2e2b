/* A plain C client of libnf4 (no Python, no torch): the header compiles as C, and the host-only calls and the
 * argument checks that return before any CUDA call behave as include/nf4.h states.  Prints "ok" on success. */
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "nf4.h"

static int failures = 0;
#define CHECK(cond)                                               \
  do {                                                            \
    if (!(cond)) {                                                \
      fprintf(stderr, "failed: %s (line %d)\n", #cond, __LINE__); \
      ++failures;                                                 \
    }                                                             \
  } while (0)

int main(void) {
  float code[16];
  nf4_code_table(code);
  CHECK(code[0] == -1.0f && code[7] == 0.0f && code[15] == 1.0f);
  for (int i = 0; i < 15; ++i) CHECK(code[i] < code[i + 1]);
  CHECK(strcmp(nf4_status_string(NF4_ERR_MISALIGNED), "NF4_ERR_MISALIGNED") == 0);
  const int64_t n = 4096LL * 4096LL, nb = n / 64;
  CHECK(nf4_storage_bytes(n, 64, 1, 256) == (size_t)(n / 2 + nb + 4 * (nb / 256) + 4));
  nf4_stream_t s = NULL;
  /* quantize: bad sizes, block size, alignment -- all rejected on the host */
  CHECK(nf4_quantize((const void *)0x1000, NF4_F32, -1, 64, (uint8_t *)0x2000, (float *)0x3000, s) ==
        NF4_ERR_INVALID_ARG);
  CHECK(nf4_quantize((const void *)0x1000, NF4_F32, 10, 512, (uint8_t *)0x2000, (float *)0x3000, s) ==
        NF4_ERR_UNSUPPORTED);
  CHECK(nf4_quantize((const void *)0x1004, NF4_F32, 10, 64, (uint8_t *)0x2000, (float *)0x3000, s) ==
        NF4_ERR_MISALIGNED);
  CHECK(nf4_quantize((const void *)0x1000, NF4_F32, 0, 64, (uint8_t *)0x2000, (float *)0x3000, s) == NF4_OK);
  /* a weight descriptor with fp32 scales */
  nf4_weight w;
  memset(&w, 0, sizeof w);
  w.packed = (const uint8_t *)0x10000;
  w.absmax = (const float *)0x20000;
  w.rows = 256;
  w.cols = 512;
  w.blocksize = 64;
  w.dq_blocksize = 256;
  CHECK(nf4_gemv(&w, (const void *)0x30000, 9, (void *)0x40000, s) == NF4_ERR_INVALID_ARG); /* batch > 8 */
  CHECK(nf4_gemm(&w, (const void *)0x30000, 0, (void *)0x40000, NULL, 0, s) == NF4_OK);      /* m = 0 */
  CHECK(nf4_gemm_dx(&w, (const void *)0x30004, 4, (void *)0x40000, NULL, 0, s) == NF4_ERR_MISALIGNED);
  nf4_lora lora = {(const void *)0x50000, (const void *)0x60000, 8, 2.0f};
  CHECK(nf4_gemm_lora(&w, &lora, (const void *)0x30000, 4, (void *)0x40000, (void *)0x70000, 1 << 20, s) ==
        NF4_ERR_UNSUPPORTED); /* r = 8 */
  lora.r = 16;
  lora.scale = (float)INFINITY;
  CHECK(nf4_gemm_lora(&w, &lora, (const void *)0x30000, 4, (void *)0x40000, (void *)0x70000, 1 << 20, s) ==
        NF4_ERR_INVALID_ARG);
  const nf4_weight *group[5] = {&w, &w, &w, &w, &w};
  void *ys[5] = {(void *)0x40000, (void *)0x40000, (void *)0x40000, (void *)0x40000, (void *)0x40000};
  CHECK(nf4_gemv_grouped(group, 5, (const void *)0x30000, 1, ys, s) == NF4_ERR_INVALID_ARG); /* more than 4 */
  /* the multi-weight GEMV: 1..NF4_GEMV_STREAM_MAX weights, batch 1..8 */
  const void *xs[2] = {(const void *)0x30000, (const void *)0x30000};
  CHECK(nf4_gemv_stream(&w, xs, ys, 0, 1, s) == NF4_ERR_INVALID_ARG);
  CHECK(nf4_gemv_stream(&w, xs, ys, NF4_GEMV_STREAM_MAX + 1, 1, s) == NF4_ERR_INVALID_ARG);
  CHECK(nf4_gemv_stream(&w, xs, ys, 1, 9, s) == NF4_ERR_INVALID_ARG);
  /* the code book: NF4 or FP4 only */
  CHECK(nf4_quantize_typed((const void *)0x1000, NF4_F32, 10, 64, 2, (uint8_t *)0x2000, (float *)0x3000, s) ==
        NF4_ERR_INVALID_ARG);
  CHECK(nf4_quantize_typed((const void *)0x1000, NF4_F32, 0, 64, NF4_QUANT_FP4, (uint8_t *)0x2000, (float *)0x3000,
                           s) == NF4_OK);
  w.quant_type = 7;
  CHECK(nf4_dequantize(&w, (void *)0x40000, NF4_BF16, s) == NF4_ERR_INVALID_ARG);
  w.quant_type = NF4_QUANT_NF4;
  w.blocksize = 48; /* level-1 sizes: 32, 64, 128, 256 */
  CHECK(nf4_dequantize(&w, (void *)0x40000, NF4_BF16, s) == NF4_ERR_UNSUPPORTED);
  w.blocksize = 128; /* dequantize takes it; the matmuls take 64 only */
  CHECK(nf4_gemv(&w, (const void *)0x30000, 1, (void *)0x40000, s) == NF4_ERR_UNSUPPORTED);
  if (failures) return 1;
  printf("ok\n");
  return 0;
}
