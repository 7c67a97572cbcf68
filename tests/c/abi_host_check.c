/* Calls the host-side entry points of libmoe_b200.so from plain C99 through
 * include/moe.h (no device memory is touched): version and status strings, the size
 * queries, host validation of a device call, and the FP4 packer round trip.
 * Prints "ok" and exits 0 when every check holds. */
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "moe.h"

#define CHECK(c)                                                   \
  do {                                                             \
    if (!(c)) {                                                    \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c); \
      return 1;                                                    \
    }                                                              \
  } while (0)

int main(void) {
  CHECK(moe_version() >= 10000);
  CHECK(strcmp(moe_status_str(MOE_ERR_WORKSPACE), "MOE_ERR_WORKSPACE") == 0);
  /* capacity: ceil(1.25 * 256 * 2 / 8) = 80 per assignment, ceil(1.25 * 256 / 8) = 40 literal */
  CHECK(moe_capacity(256, 8, 2, 1.25, 1) == 80);
  CHECK(moe_capacity(256, 8, 2, 1.25, 0) == 40);
  CHECK(moe_rows_max(100, 8, 2, 10) == 80);
  CHECK(moe_route_workspace_bytes(8192, 2048, 64) > 0);
  CHECK(moe_workspace_bytes(8192, 2048, 64, 8) >= moe_histogram_scan_workspace_bytes(8192, 8, 64));
  /* a device call rejected on the host: null x, nothing launched */
  CHECK(moe_route(NULL, MOE_BF16, NULL, NULL, NULL, NULL, 64, 128, 16, 4, MOE_SCORE_SOFTMAX, 1, 1.0f, NULL, NULL,
                  NULL, NULL, 0, NULL) == MOE_ERR_INVALID_ARG);
  /* the router's prepared split: three bf16 terms of 64 experts x 2048 */
  CHECK(moe_router_weight_bytes(2048, 64) == (size_t)3 * 64 * 2048 * 2);
  CHECK(moe_prepare_router_weight(NULL, 2048, 64, NULL, 0, NULL) == MOE_ERR_INVALID_ARG);
  /* FP4: one MXFP4 block of 32 values that E2M1 represents exactly after the 2^-3 scale */
  {
    static const float mags[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
    float w[32], back[32], ts = 0.0f;
    unsigned char codes[16], scales[1];
    int i;
    for (i = 0; i < 32; ++i) w[i] = (i & 1 ? -1.0f : 1.0f) * mags[i % 8] * 0.125f;
    CHECK(moe_fp4_block_size(MOE_FP4_MX) == 32);
    CHECK(moe_quantize_fp4_host(w, 1, 32, MOE_FP4_MX, codes, scales, NULL, 1) == MOE_OK);
    CHECK(scales[0] == 127 - 3); /* amax 0.75: floor(log2 0.75) - 2 = -3 */
    CHECK(moe_dequantize_fp4_host(codes, scales, NULL, 1, 32, MOE_FP4_MX, back, 1) == MOE_OK);
    for (i = 0; i < 32; ++i) CHECK(back[i] == w[i]);
    CHECK(moe_quantize_fp4_host(w, 1, 32, MOE_FP4_NV, codes, scales, &ts, 0) == MOE_OK);
    CHECK(fabsf(ts - 0.75f / (6.0f * 448.0f)) <= 1e-9f);
    CHECK(moe_quantize_fp4_host(w, 1, 30, MOE_FP4_MX, codes, scales, NULL, 0) == MOE_ERR_UNSUPPORTED);
  }
  printf("ok\n");
  return 0;
}
