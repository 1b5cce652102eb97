/* The C ABI used from plain C99 (no C++, no CUDA headers, no torch): the
 * header must compile as C, the library must link, and calls with bad
 * arguments must return their status before touching a device.  The
 * pointers are fake and are never dereferenced; the program runs only where
 * no kernel can launch. */
#include <stdio.h>
#include <string.h>

#include "coda.h"

static int failures = 0;

static void expect(const char* what, coda_status_t got, coda_status_t want) {
  if (got != want) {
    printf("FAIL %s: %s, expected %s\n", what, coda_status_string(got), coda_status_string(want));
    ++failures;
  }
}

int main(void) {
  const uint16_t* a = (const uint16_t*)(uintptr_t)0x10000;
  const uint16_t* b = (const uint16_t*)(uintptr_t)0x20000;
  uint16_t* c = (uint16_t*)(uintptr_t)0x30000;
  uint16_t* mis = (uint16_t*)(uintptr_t)0x30008;

  if (coda_version() < 1) {
    printf("FAIL version\n");
    ++failures;
  }
  if (coda_partial_tile_width() != 128 || coda_partial_cols(2048) != 16) {
    printf("FAIL partial layout\n");
    ++failures;
  }
  if (strcmp(coda_status_string(CODA_OK), "CODA_OK") != 0) {
    printf("FAIL status string: %s\n", coda_status_string(CODA_OK));
    ++failures;
  }
  expect("rowscale NULL out", coda_gemm_rowscale(a, b, NULL, NULL, 256, 512, 512, NULL), CODA_ERR_NULL);
  expect("rowscale bad N", coda_gemm_rowscale(a, b, NULL, c, 256, 500, 512, NULL), CODA_ERR_SHAPE);
  expect("rowscale misaligned", coda_gemm_rowscale(a, b, NULL, mis, 256, 512, 512, NULL), CODA_ERR_ALIGN);
  expect("rowscale empty batch", coda_gemm_rowscale(a, b, NULL, c, 0, 512, 512, NULL), CODA_OK);
  expect("rms_reduce eps", coda_rms_reduce((const float*)a, 16, 1, 64, -1.0f, (float*)c, NULL), CODA_ERR_SHAPE);
  expect("lmhead_ce workspace",
         coda_lmhead_ce(a, b, (const int64_t*)a, NULL, (float*)c, (float*)c, NULL, NULL, 0, 16, 64, 64, NULL),
         CODA_ERR_WORKSPACE);
  expect("qkv_rope head_dim",
         coda_gemm_qkv_rope(a, b, (const int32_t*)a, c, 16, 384, 64, 96, 192, 500000.0f, NULL), CODA_ERR_SHAPE);
  if (coda_lmhead_ce_workspace_size(8192, 128256) == 0) {
    printf("FAIL workspace size\n");
    ++failures;
  }
  if (failures == 0) printf("abi_from_c ok\n");
  return failures == 0 ? 0 : 1;
}
