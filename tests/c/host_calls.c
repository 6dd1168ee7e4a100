/* A plain C consumer of libsplitkv: host-only entry points (planners, the causal planner, argument
 * validation, status strings), so the header and the library are checked together from C. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "splitkv.h"

#define CHECK(cond)                                          \
  do {                                                       \
    if (!(cond)) {                                           \
      fprintf(stderr, "line %d: %s\n", __LINE__, #cond);     \
      return 1;                                              \
    }                                                        \
  } while (0)

int main(void) {
  CHECK(skv_version() >= 1);
  CHECK(strlen(skv_status_str(SKV_ERR_WORKSPACE)) > 0);

  /* two requests: 37 tokens (3 pages of 16) and 16 tokens (1 page); 1 and 2 query tokens */
  const int32_t qo[3] = {0, 1, 3}, kv_indptr[3] = {0, 3, 4}, last[2] = {5, 16}, kv_indices[4] = {7, 2, 9, 4};
  skv_plan_info info;
  int32_t plan[4096];
  /* a too-small buffer reports the size it needs */
  CHECK(skv_plan_paged(2, qo, kv_indptr, last, 16, 8, 2, 64, SKV_SPLIT_FIXED, 2, NULL, NULL, plan, 1, &info) ==
        SKV_ERR_WORKSPACE);
  CHECK(info.plan_words > 1 && info.plan_words <= 4096);
  CHECK(skv_plan_paged(2, qo, kv_indptr, last, 16, 8, 2, 64, SKV_SPLIT_FIXED, 2, NULL, NULL, plan, 4096, &info) ==
        SKV_OK);
  /* request 0: 1 token x 2 splits; request 1: one page, so its second split is empty */
  CHECK(info.num_partial_rows == 1 * 2 + 2 * 2 && info.num_merge_rows == 3);
  CHECK(skv_plan_paged(2, qo, kv_indptr, last, 16, 8, 3, 64, SKV_SPLIT_NONE, 0, NULL, NULL, plan, 4096, &info) ==
        SKV_ERR_INVALID); /* 3 KV heads do not divide 8 query heads */

  CHECK(skv_plan_mla(2, 4, kv_indptr, last, 16, 16, SKV_BF16, SKV_SPLIT_NONE, 0, NULL, NULL, plan, 4096, &info) ==
        SKV_OK);
  /* 16 heads x 4 tokens = 64 rows: the 64-row bf16 kernel folds all four tokens into one unit */
  CHECK(info.num_work >= 2 && info.kernel == 14 && info.q_tile == skv_mla_fold_ratio(16, 4, 64));

  /* causal tables: request 0 (L = 37, 1 token) sees everything through the prefix; request 1
   * (L = 16, 2 tokens) has a 15-token prefix and its second token adds token 15 (page 4, slot 15) */
  int32_t pi[3], px[4], pl[2], di[4], dl[3], rows[8];
  int64_t need = -1;
  CHECK(skv_causal_tables(2, qo, kv_indptr, kv_indices, last, 16, pi, px, pl, di, rows, dl, 8, &need) == SKV_OK);
  CHECK(need == 1 && pi[1] == 3 && pi[2] == 4 && pl[0] == 5 && pl[1] == 15);
  CHECK(di[0] == 0 && di[1] == 0 && di[2] == 0 && di[3] == 1 && rows[0] == 4 * 16 + 15);

  /* launches reject bad arguments before touching the device */
  skv_splice_params sp;
  memset(&sp, 0, sizeof sp);
  skv_splice_chunk ch = {0, 0, 4, 1};
  CHECK(skv_mla_splice(&sp, &ch, 1, NULL) == SKV_ERR_INVALID);
  CHECK(skv_mla_splice(&sp, &ch, 0, NULL) == SKV_OK);
  CHECK(skv_merge_states(NULL, NULL, NULL, 2, 4, 8, 64, NULL, SKV_F32, NULL, NULL) == SKV_ERR_INVALID);
  printf("ok\n");
  return 0;
}
