/* A plain C client of libfp8bs.so: the header must compile as C99 and the host-side
 * entry points (dispatch walk, census, workspace sizing, validation) must work without
 * a GPU. Prints one line per check; exits non-zero on the first failure. */
#include <stdio.h>
#include <string.h>

#include "fp8bs.h"

#define CHECK(cond, what)                      \
  do {                                         \
    if (!(cond)) {                             \
      fprintf(stderr, "FAIL: %s\n", what);     \
      return 1;                                \
    }                                          \
    printf("ok: %s\n", what);                  \
  } while (0)

int main(void) {
  int64_t padded = -1;
  int hit = -1;
  char cfg[64];
  uint64_t hits = 0, misses = 0, dh = 0, dm = 0;
  CHECK(fp8bs_version() != NULL && strlen(fp8bs_version()) > 0, "version string");
  CHECK(strlen(fp8bs_status_string(FP8BS_ERR_TIMEOUT)) > 0, "status string");
  CHECK(fp8bs_dispatch_reset_table(0) == FP8BS_OK, "empty table");
  CHECK(fp8bs_dispatch_set_row(FP8BS_OP_A8W8_BLOCKSCALE, 8, 5120, 6144, "a8w8_gemv_umma") == FP8BS_OK, "set row");
  CHECK(fp8bs_dispatch_lookup(FP8BS_OP_A8W8_BLOCKSCALE, 5, 5120, 6144, 1, &padded, &hit, cfg, sizeof cfg) ==
            FP8BS_OK && hit == 1 && padded == 8 && strcmp(cfg, "a8w8_gemv_umma") == 0,
        "M=5 served by the M=8 row");
  CHECK(fp8bs_dispatch_lookup(FP8BS_OP_A8W8_BLOCKSCALE, 17, 5120, 6144, 1, &padded, &hit, cfg, sizeof cfg) ==
            FP8BS_OK && hit == 0 && padded == 0,
        "M=17 misses");
  CHECK(fp8bs_dispatch_stats(FP8BS_OP_A8W8_BLOCKSCALE, &hits, &misses, &dh, &dm) == FP8BS_OK && hits >= 1 &&
            misses >= 1,
        "census counts");
  CHECK(fp8bs_dispatch_set_row(FP8BS_OP_A8W8_BLOCKSCALE, 64, 5120, 6144, "a8w8_gemv_umma") ==
            FP8BS_ERR_UNSUPPORTED,
        "weight-streaming row refused above M=32");
  CHECK(fp8bs_dispatch_reset_table(1) == FP8BS_OK, "built-in table restored");
  CHECK(fp8bs_workspace_bytes(FP8BS_OP_A8W8_BLOCKSCALE, 1, 5120, 6144) > 0, "decode needs a workspace");
  CHECK(fp8bs_gemm_a8w8_blockscale(NULL, NULL, NULL, NULL, NULL, 1, 5120, 6144, NULL, 0, NULL) ==
            FP8BS_ERR_INVALID_ARG,
        "null pointers rejected before any launch");
  return 0;
}
