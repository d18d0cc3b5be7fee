/* A plain C99 consumer of libfp8attn: it includes only include/fp8attn.h and
 * calls the entry points that do their work (or reject their arguments) on
 * the host, so it runs without a GPU.  The selector examples are the ones the
 * vLLM-Omni "Quantized KV Cache" page gives in its parameters table
 * ("0,1,4-6" and "0-2,10"). */
#include <stdio.h>
#include <string.h>

#include "fp8attn.h"

static int fails = 0;
#define CHECK(c)                                                        \
  do {                                                                  \
    if (!(c)) {                                                         \
      printf("FAIL line %d: %s\n", __LINE__, #c);                       \
      ++fails;                                                          \
    }                                                                   \
  } while (0)

static int mask_is(const uint8_t* m, int n, const int* on, int n_on) {
  int i, j;
  for (i = 0; i < n; ++i) {
    int want = 0;
    for (j = 0; j < n_on; ++j)
      if (on[j] == i) want = 1;
    if ((m[i] != 0) != want) return 0;
  }
  return 1;
}

int main(void) {
  uint8_t mask[12];
  static const int sel_a[] = {0, 1, 4, 5, 6};
  static const int sel_b[] = {0, 1, 2, 10};
  fp8attn_ctx* ctx = (fp8attn_ctx*)0;

  CHECK(fp8attn_ring_length() == 16);
  CHECK(fp8attn_workspace_bytes(0) == 0);
  CHECK(fp8attn_workspace_bytes(3) == 256 + 3 * 320);
  CHECK(strcmp(fp8attn_status_string(FP8ATTN_OK), "ok") == 0);
  CHECK(strcmp(fp8attn_status_string(12345), "unknown status") == 0);

  CHECK(fp8attn_parse_selector("0,1,4-6", 12, mask) == FP8ATTN_OK);
  CHECK(mask_is(mask, 12, sel_a, 5));
  CHECK(fp8attn_parse_selector("0-2,10", 12, mask) == FP8ATTN_OK);
  CHECK(mask_is(mask, 12, sel_b, 4));
  CHECK(fp8attn_parse_selector((const char*)0, 12, mask) == FP8ATTN_OK);
  CHECK(mask_is(mask, 12, sel_a, 0));
  CHECK(fp8attn_parse_selector("6-4", 12, mask) != FP8ATTN_OK);
  CHECK(fp8attn_parse_selector("12", 12, mask) != FP8ATTN_OK);

  /* argument checks that return before any CUDA call */
  CHECK(fp8attn_create(0, (void*)256, 1 << 20, (void*)0, &ctx) == FP8ATTN_ERR_INVALID);
  CHECK(ctx == (fp8attn_ctx*)0);
  CHECK(fp8attn_select_mode((const fp8attn_ctx*)0, (const uint8_t*)0, 0) == -1);
  CHECK(fp8attn_regroup_heads((const void*)0, (void*)0, 0, 8, 2, 256, 1, (void*)0) ==
        FP8ATTN_OK);
  CHECK(fp8attn_regroup_heads((const void*)4096, (void*)(1 << 20), 4, 8, 3, 256, 1,
                              (void*)0) == FP8ATTN_ERR_INVALID);
  CHECK(fp8attn_varlen_fwd((const void*)0, (const void*)0, (const void*)0, (const int32_t*)16,
                           1, 8, 0, 8, 128, (const float*)0, 0.0f, (void*)0, (int32_t*)0,
                           (void*)0) == FP8ATTN_OK);
  CHECK(fp8attn_varlen_fwd((const void*)16, (const void*)16, (const void*)16,
                           (const int32_t*)16, 1, 8, 8, 8, 64, (const float*)16, 0.0f,
                           (void*)16, (int32_t*)0, (void*)0) == FP8ATTN_ERR_UNSUPPORTED);
  /* work schedules: the three named ones pass the checks (zero tokens), others
   * are invalid */
  CHECK(fp8attn_varlen_fwd_sched((const void*)0, (const void*)0, (const void*)0,
                                 (const int32_t*)16, 1, 8, 0, 8, 128, (const float*)0, 0.0f,
                                 FP8ATTN_P_LINEAR_LOG, FP8ATTN_SCHED_SPLIT, (void*)0,
                                 (int32_t*)0, (void*)0) == FP8ATTN_OK);
  CHECK(fp8attn_varlen_fwd_sched((const void*)0, (const void*)0, (const void*)0,
                                 (const int32_t*)16, 1, 8, 0, 8, 128, (const float*)0, 0.0f,
                                 FP8ATTN_P_EXP2, 7, (void*)0, (int32_t*)0,
                                 (void*)0) == FP8ATTN_ERR_INVALID);
  /* the grouped cast: DYNAMIC and a group count that does not divide the
   * heads are refused before the context is touched */
  CHECK(fp8attn_quantize_qkv_grouped((fp8attn_ctx*)0, 0, FP8ATTN_DYNAMIC, (const void*)16,
                                     (const void*)16, (const void*)16, 1024, 128,
                                     (const int32_t*)0, (const int32_t*)16, 1, 8, 8, 8, 128, 2,
                                     (void*)16, (void*)16, (void*)16,
                                     (void*)0) == FP8ATTN_ERR_INVALID);
  CHECK(fp8attn_quantize_qkv_grouped((fp8attn_ctx*)0, 0, FP8ATTN_RING, (const void*)16,
                                     (const void*)16, (const void*)16, 1024, 128,
                                     (const int32_t*)0, (const int32_t*)16, 1, 8, 8, 8, 128, 3,
                                     (void*)16, (void*)16, (void*)16,
                                     (void*)0) == FP8ATTN_ERR_INVALID);
  /* the static cast inside attention: a missing context is refused before
   * anything else is looked at */
  CHECK(fp8attn_varlen_fwd_static((fp8attn_ctx*)0, 0, (const void*)16, (const void*)16,
                                  (const void*)16, 1024, 128, (const int32_t*)16, 1, 8, 8, 8,
                                  128, 0.0f, FP8ATTN_P_LINEAR_LOG, (void*)16,
                                  (void*)0) == FP8ATTN_ERR_INVALID);

  /* the static scale map: parse (with the margin), format, apply_margin */
  {
    static const char text[] =
        "{\"visual.blocks.0.attn.attn\": {\"q\": 224, \"k\": 198, \"v\": 210},\n"
        " \"visual.blocks.1.attn.attn\": {\"q_scale\": 218, \"k_scale\": 195, \"v_scale\": 207}}";
    char names[2 * FP8ATTN_SCALE_NAME_MAX];
    float vals[6], again[6];
    int n = -1;
    size_t need = 0;
    char out[512];
    CHECK(fp8attn_scale_map_parse(text, sizeof(text) - 1, 1.0f, 2, names, vals, &n) == FP8ATTN_OK);
    CHECK(n == 2 && vals[0] == 224.0f && vals[4] == 195.0f);
    CHECK(strcmp(names + FP8ATTN_SCALE_NAME_MAX, "visual.blocks.1.attn.attn") == 0);
    CHECK(fp8attn_scale_map_parse(text, sizeof(text) - 1, 1.0f, 1, names, vals, &n) ==
          FP8ATTN_ERR_INVALID);
    CHECK(fp8attn_scale_map_parse(text, sizeof(text) - 1, 1.5f, 2, names, vals, &n) == FP8ATTN_OK);
    CHECK(vals[0] == 336.0f && vals[5] == 310.5f);
    CHECK(fp8attn_scale_map_format(2, names, vals, (char*)0, 0, &need) == FP8ATTN_ERR_INVALID);
    CHECK(need > 0 && need <= sizeof(out));
    CHECK(fp8attn_scale_map_format(2, names, vals, out, sizeof(out), &need) == FP8ATTN_OK);
    CHECK(fp8attn_scale_map_parse(out, strlen(out), 1.0f, 2, names, again, &n) == FP8ATTN_OK);
    CHECK(n == 2 && memcmp(vals, again, sizeof(vals)) == 0);
    CHECK(fp8attn_apply_margin(vals, 6, 1.5f, again) == FP8ATTN_OK && again[0] == 504.0f);
    CHECK(fp8attn_apply_margin(vals, 6, 0.0f, again) == FP8ATTN_ERR_INVALID);
  }

  if (fails)
    printf("FAILED (%d)\n", fails);
  else
    printf("ok\n");
  return fails != 0;
}
