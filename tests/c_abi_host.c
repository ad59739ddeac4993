/* A plain C user of libpagedattn.so: host-side calls only (block manager,
 * prefix reuse, the shared-prefix splitter, status strings), so it runs
 * without a GPU.  Prints "ok" and exits 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "pagedattn.h"

#define CHECK(c)                                                   \
  do {                                                             \
    if (!(c)) {                                                    \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c); \
      return 1;                                                    \
    }                                                              \
  } while (0)

int main(void) {
  int32_t tables[4 * 4], lens[4];
  int64_t ids[4] = {10, 11, 12, 13};
  int32_t prompt[10] = {1, 2, 3, 4, 5, 6, 7, 8, 9, 10};
  int32_t pt[2 * 4], pl[2], tt[4 * 4], tl[4];
  int64_t slot;
  int32_t src, dst;
  int cached = -1;
  int i;
  pa_bm* bm = pa_bm_create(32, 4, 0);

  CHECK(bm != NULL);
  CHECK(strcmp(pa_status_string(PA_OK), "ok") == 0);
  /* two samples of one prompt: fork shares, the first append copies */
  CHECK(pa_bm_add_seq(bm, 10, 6) == PA_OK);
  CHECK(pa_bm_fork(bm, 10, 11) == PA_OK);
  CHECK(pa_bm_refcount(bm, 0) == 2 && pa_bm_refcount(bm, 1) == 2);
  CHECK(pa_bm_append_slot(bm, 10, &slot, &src, &dst) == PA_OK);
  CHECK(src == 1 && dst >= 0 && slot == (int64_t)dst * 4 + 2);
  CHECK(pa_bm_append_slot(bm, 11, &slot, &src, &dst) == PA_OK);
  CHECK(src == -1 && dst == -1 && slot == 1 * 4 + 2);
  /* two requests that begin alike: the second takes over two full blocks */
  CHECK(pa_bm_add_seq_tokens(bm, 12, prompt, 10, &cached) == PA_OK && cached == 0);
  CHECK(pa_bm_add_seq_tokens(bm, 13, prompt, 9, &cached) == PA_OK && cached == 8);
  CHECK(pa_bm_num_cached_blocks(bm) == 2);
  CHECK(pa_bm_export(bm, ids, 4, tables, 4, lens) == PA_OK);
  CHECK(lens[0] == 7 && lens[1] == 7 && lens[2] == 10 && lens[3] == 9);
  CHECK(tables[2 * 4 + 0] == tables[3 * 4 + 0] && tables[2 * 4 + 1] == tables[3 * 4 + 1]);
  /* groups of two: (10, 11) share block 0, (12, 13) share two blocks */
  CHECK(pa_split_shared_prefix(tables, lens, 4, 4, 4, 2, pt, 4, pl, tt, 4, tl) == PA_OK);
  CHECK(pl[0] == 4 && pl[1] == 8);
  CHECK(pt[0] == 0 && pt[1] == -1 && pt[4] == tables[2 * 4] && pt[5] == tables[2 * 4 + 1]);
  CHECK(tl[0] == 3 && tl[1] == 3 && tl[2] == 2 && tl[3] == 1);
  for (i = 0; i < 4; ++i) CHECK(pa_bm_free_seq(bm, ids[i]) == PA_OK);
  CHECK(pa_bm_num_free(bm) == 32);
  CHECK(pa_bm_free_seq(bm, 10) == PA_ERR_NO_SEQ);
  pa_bm_destroy(bm);
  /* argument errors come back before any device work */
  CHECK(pa_paged_attn_decode(NULL, NULL, NULL, NULL, NULL, NULL, 1.f, 4, 8, 64, 4, 8, 64, PA_F16,
                             NULL, 0, NULL, NULL) == PA_ERR_INVALID);
  printf("ok\n");
  return 0;
}
