/* Plain C99 client of include/dq.h: compiled and run by tests/test_abi.py
 * (no GPU needed).  Every call below returns before any device work: size
 * queries, or arguments the library must reject with its documented status. */
#include <stdint.h>
#include <stdio.h>

#include "dq.h"

#define CHECK(cond)                                        \
  do {                                                     \
    if (!(cond)) {                                         \
      fprintf(stderr, "check failed: %s\n", #cond);        \
      return 1;                                            \
    }                                                      \
  } while (0)

int main(void) {
  void* fake = (void*)(uintptr_t)0x1000;
  void* ws = (void*)(uintptr_t)0x2000;
  const void* Ws[2] = {fake, fake};
  float* fs[2] = {(float*)fake, (float*)fake};
  int64_t m[2] = {64, 64}, n[2] = {64, 40};

  CHECK(dq_version() >= 200);
  CHECK(dq_native_group(DQ_NVFP4) == 16 && dq_native_group(DQ_MXFP4) == 32 &&
        dq_native_group(DQ_MXINT4) == 32 && dq_native_group(DQ_INT4) == 64);
  CHECK(dq_scales_bytes(300, 5120, DQ_NVFP4, 16) == (size_t)(3 * 80 * 512));
  CHECK(dq_scales_bytes(10, 256, DQ_INT4, 128) == 40);
  CHECK(dq_solve_batched_workspace_size(3, 7) == 3 * dq_solve_workspace_size(7));
  CHECK(dq_status_string(DQ_OK) != NULL);

  CHECK(dq_solve_scales(NULL, DQ_BF16, 64, 64, DQ_NVFP4, 16, 5, (float*)fake, (float*)fake,
                        (float*)fake, NULL, ws, 4096, NULL) == DQ_ERR_ARG);
  CHECK(dq_solve_scales_ex(fake, DQ_BF16, 64, 64, DQ_NVFP4, 16, 5,
                           DQ_SOLVE_ALPHA_ONLY | DQ_SOLVE_BETA_ONLY, NULL, NULL, (float*)fake,
                           (float*)fake, (float*)fake, NULL, ws, 4096, NULL) == DQ_ERR_ARG);
  CHECK(dq_solve_scales_batched(2, Ws, DQ_BF16, m, n, DQ_NVFP4, 16, 5, 0, fs, fs, fs, NULL, ws,
                                4096, NULL) == DQ_ERR_ARG);
  CHECK(dq_quantize_act(fake, DQ_BF16, 4, 48, NULL, DQ_NVFP4, 16, (uint8_t*)fake, fake,
                        (float*)fake, NULL) == DQ_ERR_ARG);
  CHECK(dq_act_quant_error(fake, DQ_BF16, 4, 64, NULL, DQ_NVFP4, 16, (const uint8_t*)fake, fake,
                           NULL, (double*)fake, NULL) == DQ_ERR_ARG);
  CHECK(dq_w4a4_linear((const uint8_t*)fake, (const uint8_t*)fake, (const float*)fake,
                       (const uint8_t*)fake, (const uint8_t*)fake, (const float*)fake, NULL, fake,
                       DQ_BF16, 16, 128, 256, DQ_INT4, NULL) == DQ_ERR_UNSUPPORTED);
  printf("c abi ok\n");
  return 0;
}
