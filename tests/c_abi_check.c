/*
 * A plain C caller of the library: includes only include/lkv.h, links liblkv.so, and exercises
 * the host-only entry points (work partition, workspace and FP8 row sizes, argument checks),
 * none of which makes a CUDA call.  Built and run by tests/test_c_abi.py; exits 0 when every
 * check holds and prints the first failing check otherwise.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "lkv.h"

static int failures = 0;

#define CHECK(cond)                                                  \
  do {                                                               \
    if (!(cond)) {                                                   \
      fprintf(stderr, "check failed (line %d): %s\n", __LINE__, #cond); \
      ++failures;                                                    \
    }                                                                \
  } while (0)

int main(void) {
  CHECK(lkv_version() >= 100);
  for (int s = 0; s <= 5; ++s) CHECK(lkv_status_string(s) != NULL && strlen(lkv_status_string(s)) > 0);

  /* work partition: one range per request at B = 64 (MLA), groups in lockstep (GQLA / GTA) */
  CHECK(lkv_plan_ranges(0, 64, 1, 1, 148) == 64);
  CHECK(lkv_plan_ranges(1, 64, 2, 8, 148) == 144);
  CHECK(lkv_plan_ranges(3, 64, 2, 8, 148) == 144);
  CHECK(lkv_plan_ranges(7, 64, 2, 8, 148) == -1);

  /* segments of two MLA requests (300 and 600 keys, 256-key tiles) over 3 ranges: every tile once */
  {
    const int32_t cu[3] = {0, 300, 900};
    int32_t rec[8 * 32];
    const int n = lkv_plan_segments(0, cu, 2, 1, 1, 3, rec, 32);
    CHECK(n > 0 && n <= 32);
    int tiles = 0;
    for (int i = 0; i < n && i < 32; ++i) {
      const int32_t* r = rec + 8 * i;
      CHECK(r[0] >= 0 && r[0] < 3);             /* range */
      CHECK(r[1] >= 0 && r[1] < 2);             /* request */
      CHECK(r[3] >= 0 && r[3] < r[4]);          /* tile_lo < tile_hi */
      tiles += r[4] - r[3];
    }
    CHECK(tiles == 2 + 3);
    CHECK(lkv_plan_segments(0, NULL, 2, 1, 1, 3, rec, 32) == -1);
  }

  /* workspace sizes: positive for valid shapes, 0 for an unknown kind */
  CHECK(lkv_mla_decode_workspace_size(64, 1, 128, 512, 148) > 0);
  CHECK(lkv_group_decode_workspace_size(1, 64, 2, 128, 8, 128, 148) > 0);
  CHECK(lkv_group_decode_workspace_size(3, 64, 2, 128, 8, 128, 148) ==
        lkv_group_decode_workspace_size(1, 64, 2, 128, 8, 128, 148));
  CHECK(lkv_group_decode_workspace_size(9, 64, 2, 128, 8, 128, 148) == 0);

  /* FP8 cache rows: 512 codes + 16 bytes of scale + 64 bf16 RoPE values */
  CHECK(lkv_fp8_cache_row_bytes(512, 64) == 656);
  CHECK(lkv_fp8_cache_row_bytes(500, 64) == 0);

  /* argument errors are found before any CUDA call */
  {
    void* p = (void*)(uintptr_t)(1u << 20);
    const int32_t* cu = (const int32_t*)(uintptr_t)(1u << 21);
    float* f = (float*)(uintptr_t)(1u << 20);
    CHECK(lkv_mla_absorbed_decode(NULL, p, p, 576, p, 576, 1000, cu, 2, 1, 128, 512, 64, 0.04f, LKV_BF16, p, f, p,
                                  1u << 30, NULL) == LKV_ERR_INVALID_ARG);
    CHECK(lkv_mla_absorbed_decode(p, p, p, 576, p, 576, 1000, cu, 2, 3, 128, 512, 64, 0.04f, LKV_BF16, p, f, p,
                                  1u << 30, NULL) == LKV_ERR_UNSUPPORTED);
    CHECK(lkv_gqla_group_decode(p, p, p, 1024, p, 1024, p, 64, 1000, cu, 2, 2, 128, 3, 128, 64, 0.07f, LKV_BF16,
                                p, f, p, 1u << 30, NULL) == LKV_ERR_INVALID_ARG);
    CHECK(lkv_gta_group_decode(p, p, p, 1000, p, 1088, 1000, cu, 2, 2, 128, 8, 128, 64, 0.07f, LKV_BF16, p, f, p,
                               1u << 30, NULL) == LKV_ERR_INVALID_ARG);
    CHECK(lkv_gla_group_decode(p, p, p, 576, p, 576, 1000, cu, 2, 1, 128, 2, 256, 64, -1.0f, LKV_BF16, p, f, p,
                               1u << 30, NULL) == LKV_ERR_INVALID_ARG);
    CHECK(lkv_quantize_latent_fp8(p, 570, p, 656, 4, 512, 64, NULL) == LKV_ERR_INVALID_ARG);
    CHECK(lkv_absorb_query(p, p, p, 4, 6, 4, 8, 16, LKV_BF16, NULL) == LKV_ERR_INVALID_ARG);
    CHECK(lkv_output_projection(p, p, NULL, 4, 16, 8, LKV_FP32, NULL) == LKV_ERR_INVALID_ARG);
  }

  if (failures) return 1;
  printf("ok\n");
  return 0;
}
