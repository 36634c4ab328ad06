/* Plain C (C99) client of include/attn.h: it compiles the header as C, links the library
 * and calls the host-only entry points (no CUDA call, no GPU needed). Checks, for two
 * sequences of 300 and 200 rows:
 *   - CAUSAL tile classes and the visible-pair count (closed form L (L + 1) / 2 per
 *     sequence);
 *   - the same mask written as one CAUSAL range per sequence gives the same classes;
 *   - a dry-run plan's statistics agree with the classes;
 *   - an invalid problem (hq not a multiple of hkv) is rejected with a status, not a crash.
 * Prints "ok" and exits 0 on success; prints the failed check and exits 1 otherwise. */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "attn.h"

#define CHECK(cond)                                                  \
  do {                                                               \
    if (!(cond)) {                                                   \
      printf("check failed at line %d: %s\n", __LINE__, #cond);    \
      return 1;                                                      \
    }                                                                \
  } while (0)

static int tiles_of(int lq, int lk) { return ((lq + 127) / 128) * ((lk + 127) / 128); }

int main(void) {
  const int32_t cu[3] = {0, 300, 500};
  attn_problem_t p;
  memset(&p, 0, sizeof(p));
  p.batch = 2;
  p.hq = 4;
  p.hkv = 2;
  p.head_dim = 128;
  p.cu_seqlens_q = cu;
  p.cu_seqlens_k = cu;

  attn_mask_desc_t causal;
  memset(&causal, 0, sizeof(causal));
  causal.kind = ATTN_MASK_CAUSAL;

  size_t need = 0;
  int64_t pairs = 0;
  CHECK(attn_classify_host(&p, &causal, NULL, 0, &need, &pairs) == ATTN_OK);
  CHECK(need == (size_t)(tiles_of(300, 300) + tiles_of(200, 200)));
  CHECK(pairs == 300LL * 301 / 2 + 200LL * 201 / 2);
  uint8_t* cls = (uint8_t*)malloc(need);
  CHECK(cls != NULL);
  CHECK(attn_classify_host(&p, &causal, cls, need, NULL, NULL) == ATTN_OK);
  /* sequence 0 (3 x 3 tiles, the last row and column 44 wide): diagonal tiles partial (2),
   * above the diagonal empty (0), below it full (1); classes are taken over each tile's
   * valid rectangle, so the 44 x 128 tiles of the last row are full too */
  CHECK(cls[0] == 2 && cls[1] == 0 && cls[2] == 0);
  CHECK(cls[3] == 1 && cls[4] == 2 && cls[5] == 0);
  CHECK(cls[6] == 1 && cls[7] == 1 && cls[8] == 2);

  /* the same mask as one CAUSAL range per sequence */
  attn_range_t ranges[2];
  memset(ranges, 0, sizeof(ranges));
  ranges[0].q_end = 300; ranges[0].k_end = 300; ranges[0].type = ATTN_RANGE_CAUSAL;
  ranges[1].q_end = 200; ranges[1].k_end = 200; ranges[1].type = ATTN_RANGE_CAUSAL;
  const int32_t cu_ranges[3] = {0, 1, 2};
  attn_mask_desc_t rm;
  memset(&rm, 0, sizeof(rm));
  rm.kind = ATTN_MASK_RANGES;
  rm.ranges = ranges;
  rm.cu_ranges = cu_ranges;
  uint8_t* cls2 = (uint8_t*)malloc(need);
  CHECK(cls2 != NULL);
  int64_t pairs2 = 0;
  CHECK(attn_classify_host(&p, &rm, cls2, need, NULL, &pairs2) == ATTN_OK);
  CHECK(pairs2 == pairs && memcmp(cls, cls2, need) == 0);

  /* dry-run statistics */
  attn_plan_stats_t st;
  memset(&st, 0, sizeof(st));
  CHECK(attn_plan_dry_run(&p, &causal, 148, &st) == ATTN_OK);
  int64_t e = 0, f = 0, q = 0;
  for (size_t i = 0; i < need; ++i) {
    e += cls[i] == 0;
    f += cls[i] == 1;
    q += cls[i] == 2;
  }
  CHECK(st.unmasked_pairs == pairs);
  CHECK(st.tiles_empty == e && st.tiles_full == f && st.tiles_partial == q);
  CHECK(st.work_items > 0 && st.jobs > 0 && st.ctas > 0 && st.workspace_bytes > 0);

  /* errors are statuses */
  p.hq = 3;
  CHECK(attn_classify_host(&p, &causal, NULL, 0, &need, NULL) == ATTN_ERR_INVALID_ARG);
  CHECK(attn_plan_dry_run(&p, &causal, 148, &st) == ATTN_ERR_INVALID_ARG);
  CHECK(attn_status_string(ATTN_ERR_INVALID_ARG) != NULL);

  free(cls);
  free(cls2);
  printf("ok\n");
  return 0;
}
