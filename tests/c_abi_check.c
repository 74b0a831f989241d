/* A plain C99 client of libnvfp4.so: it includes only include/nvfp4.h and calls the
 * host-only parts of the C ABI (sizes, status names, argument validation), so that
 * the boundary is checked from C, without Python or a GPU.  Built and run by
 * tests/test_library_host.py; prints "ok" and exits 0 when every check holds. */
#include <stdio.h>
#include <string.h>

#include "nvfp4.h"

static int failures = 0;

static void check(int cond, const char *what) {
  if (!cond) {
    fprintf(stderr, "FAILED: %s\n", what);
    ++failures;
  }
}

int main(void) {
  static unsigned char buf[64] __attribute__((aligned(16)));
  check(nvfp4_scale_bytes(200, 80) == 2048, "scale bytes of 200 x 80");
  check(nvfp4_scale_bytes(8192, 5120) == 2621440, "scale bytes of 8192 x 5120");
  check(nvfp4_scale_bytes(0, 64) == 0, "scale bytes of an empty tensor");
  check(nvfp4_scale_bytes(4, 24) == -1, "k not a multiple of 16");
  check(strcmp(nvfp4_status_string(NVFP4_ERR_INVALID_ARGUMENT), "NVFP4_ERR_INVALID_ARGUMENT") == 0,
        "status name");
  /* invalid arguments are rejected before any device work */
  check(nvfp4_quantize(buf, 4, 24, (const float *)buf, buf, buf, NULL) == NVFP4_ERR_INVALID_ARGUMENT,
        "quantize with k % 16 != 0");
  check(nvfp4_gemm(buf, buf, buf, buf, (const float *)buf, NULL, buf, 128, 250, 256, NULL) ==
            NVFP4_ERR_INVALID_ARGUMENT,
        "gemm with n % 8 != 0");
  /* empty problems are no-ops */
  check(nvfp4_quantize(NULL, 0, 32, NULL, NULL, NULL, NULL) == NVFP4_OK, "empty quantize");
  check(nvfp4_gemm(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, 256, 256, NULL) == NVFP4_OK, "empty gemm");
  if (failures) return 1;
  printf("ok\n");
  return 0;
}
