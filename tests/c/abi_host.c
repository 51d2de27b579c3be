/* The C ABI from plain C99 (no Python, no GPU): the host-only block manager on the
 * framework-overview flowchart of "PagedAttention - Efficient Memory Management for
 * LLM Serving with vLLM" (the scenarios of tests/golden/block_manager_flowchart.json:
 * sequence 1 holds P3, P7, P1, sequence 2 holds the shared P3 and P5; a write into a
 * shared P3 copies it to P9), plus host-side argument checks and the pure host
 * queries.  Exit status 0 when every check holds; each failure is printed. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "pagedkv.h"

static int failures = 0;

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

static void flowchart_tables(void) {
  const int32_t order[10] = {3, 7, 1, 5, 9, 0, 2, 4, 6, 8};
  pkv_block_manager* bm = pkv_bm_create(10, 16, order);
  CHECK(bm != NULL);
  CHECK(pkv_bm_add_sequence(bm, 2, 16) == PKV_OK);
  CHECK(pkv_bm_fork(bm, 2, 1) == PKV_OK);
  int64_t slot, pairs[2];
  int np;
  for (int i = 0; i < 21; ++i) {
    const int64_t s = 1;
    CHECK(pkv_bm_append_tokens(bm, &s, 1, &slot, pairs, &np) == PKV_OK && np == 0);
  }
  for (int i = 0; i < 4; ++i) {
    const int64_t s = 2;
    CHECK(pkv_bm_append_tokens(bm, &s, 1, &slot, pairs, &np) == PKV_OK && np == 0);
  }
  int32_t row[4];
  int64_t tokens = 0;
  CHECK(pkv_bm_block_table(bm, 1, row, 4, &tokens) == 3);
  CHECK(row[0] == 3 && row[1] == 7 && row[2] == 1 && row[3] == -1 && tokens == 37);
  CHECK(pkv_bm_block_table(bm, 2, row, 4, &tokens) == 2);
  CHECK(row[0] == 3 && row[1] == 5 && tokens == 20);
  CHECK(pkv_bm_ref_count(bm, 3) == 2 && pkv_bm_ref_count(bm, 7) == 1 && pkv_bm_ref_count(bm, 5) == 1);
  CHECK(pkv_bm_num_free(bm) == 6);
  /* freeing both sequences returns every block */
  CHECK(pkv_bm_free_sequence(bm, 1) == PKV_OK && pkv_bm_free_sequence(bm, 2) == PKV_OK);
  CHECK(pkv_bm_num_free(bm) == 10);
  CHECK(pkv_bm_free_sequence(bm, 2) == PKV_ESEQ);
  pkv_bm_destroy(bm);
}

static void flowchart_copy_on_write(void) {
  const int32_t order[10] = {3, 9, 0, 1, 2, 4, 5, 6, 7, 8};
  pkv_block_manager* bm = pkv_bm_create(10, 16, order);
  CHECK(bm != NULL);
  CHECK(pkv_bm_add_sequence(bm, 1, 10) == PKV_OK);
  CHECK(pkv_bm_fork(bm, 1, 2) == PKV_OK);
  int64_t slot = -1, pairs[2] = {-1, -1};
  int np = -1;
  const int64_t s2 = 2, s1 = 1;
  CHECK(pkv_bm_append_tokens(bm, &s2, 1, &slot, pairs, &np) == PKV_OK);
  CHECK(np == 1 && pairs[0] == 3 && pairs[1] == 9 && slot == 9 * 16 + 10);
  CHECK(pkv_bm_append_tokens(bm, &s1, 1, &slot, pairs, &np) == PKV_OK);
  CHECK(np == 0 && slot == 3 * 16 + 10);
  CHECK(pkv_bm_ref_count(bm, 3) == 1 && pkv_bm_ref_count(bm, 9) == 1);
  /* swap sequence 2 out and back in: it keeps its length, takes fresh blocks */
  int64_t blocks[4];
  int nb = 0;
  CHECK(pkv_bm_swap_out(bm, 2, blocks, 4, &nb) == PKV_OK && nb == 1 && blocks[0] == 9);
  CHECK(pkv_bm_ref_count(bm, 9) == 0);
  CHECK(pkv_bm_swap_in(bm, 2, blocks, 4, &nb) == PKV_OK && nb == 1);
  int32_t row[2];
  int64_t tokens = 0;
  CHECK(pkv_bm_block_table(bm, 2, row, 2, &tokens) == 1 && row[0] == blocks[0] && tokens == 11);
  pkv_bm_destroy(bm);
}

static void rejections(void) {
  const int32_t dup[3] = {0, 0, 1};
  CHECK(pkv_bm_create(0, 16, NULL) == NULL);
  CHECK(pkv_bm_create(3, 16, dup) == NULL);
  pkv_block_manager* bm = pkv_bm_create(2, 4, NULL);
  CHECK(pkv_bm_add_sequence(bm, 7, 9) == PKV_ENOMEM); /* needs 3 blocks */
  CHECK(pkv_bm_num_free(bm) == 2);                    /* nothing taken */
  pkv_bm_destroy(bm);
  /* host-side argument checks run before any CUDA call */
  CHECK(kv_block_copy((void*)0x10000, (void*)0x10000, NULL, 1, 2, 64, 16, 4, PKV_F16, NULL) == PKV_EINVAL);
  CHECK(kv_cache_append((void*)0x10000, (void*)0x10000, (void*)0x10000, (void*)0x10000, (void*)0x10004, 1, 2, 64,
                        16, 4, PKV_F16, NULL) == PKV_EALIGN);
  CHECK(pkv_selftest_wait_timeout(0, NULL) == PKV_EINVAL);
}

static void queries(void) {
  CHECK(pkv_abi_version() == 1);
  for (int code = -10; code <= 0; ++code) CHECK(pkv_strerror(code) != NULL && strlen(pkv_strerror(code)) > 0);
  /* batch-256 layer, 40 heads x 128, contexts up to 2048, B = 16: no split, counters + 8-byte unit entries */
  CHECK(paged_attn_decode_workspace_size(256, 40, 128, 16, 128, 0) == 16 + 256 * 8);
  CHECK(paged_attn_decode_partition_tokens(256, 40, 128, 16, 128, 0) == 2048);
  CHECK(paged_attn_decode_workspace_size(4, 2, 96, 16, 3, 0) == (size_t)-1); /* head_dim 96 */
}

int main(void) {
  flowchart_tables();
  flowchart_copy_on_write();
  rejections();
  queries();
  if (failures) {
    fprintf(stderr, "%d check(s) failed\n", failures);
    return 1;
  }
  printf("C ABI checks passed\n");
  return 0;
}
