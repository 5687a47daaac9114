/* Plain C (C11) client of libpagedattn: include/pa.h compiles as C, and the host
 * allocator works through the C ABI alone, with no GPU and no Python.  The sequence of
 * calls follows the copy-on-write story of the pages ("深入解析 PagedAttention",
 * 多序列共享; "PagedAttention" concept card, 实现要点): a 10-token sequence in blocks of 4
 * is forked, the child's first append copies the shared partial block, the parent then
 * writes in place, and freeing returns blocks at refcount 0.  Prints "ok" and exits 0
 * when every check holds; otherwise names the first failed check and exits 1. */
#include <stdio.h>
#include <string.h>

#include "pa.h"

#define CHECK(cond)                                                 \
  do {                                                              \
    if (!(cond)) {                                                  \
      printf("failed: %s (line %d)\n", #cond, __LINE__);            \
      return 1;                                                     \
    }                                                               \
  } while (0)

int main(void) {
  pa_allocator* a = NULL;
  CHECK(pa_alloc_create(4, 4, 0, &a) == PA_OK && a != NULL);
  CHECK(pa_alloc_num_free(a) == 4);

  /* 10 tokens in blocks of 4: three blocks, two empty slots in the last */
  CHECK(pa_alloc_add_seq(a, 0, 10) == PA_OK);
  int32_t table[8];
  int n = 0, ntok = 0;
  CHECK(pa_alloc_block_table(a, 0, table, 8, &n, &ntok) == PA_OK);
  CHECK(n == 3 && ntok == 10 && table[0] == 0 && table[1] == 1 && table[2] == 2);
  CHECK(pa_alloc_internal_waste_slots(a) == 2);

  /* fork: the child shares all three blocks */
  CHECK(pa_alloc_fork(a, 0, 1) == PA_OK);
  CHECK(pa_alloc_refcount(a, 0) == 2 && pa_alloc_refcount(a, 2) == 2);
  CHECK(pa_alloc_fork(a, 0, 1) == PA_ERR_EXISTS);

  /* the child appends first: the shared partial block 2 is copied to the free block 3 */
  int64_t slot = -1;
  int32_t src = 0, dst = 0;
  CHECK(pa_alloc_append_slot(a, 1, &slot, &src, &dst) == PA_OK);
  CHECK(src == 2 && dst == 3 && slot == 3 * 4 + 2);
  CHECK(pa_alloc_refcount(a, 2) == 1 && pa_alloc_refcount(a, 3) == 1);

  /* the parent then writes in place */
  CHECK(pa_alloc_append_slot(a, 0, &slot, &src, &dst) == PA_OK);
  CHECK(src == -1 && dst == -1 && slot == 2 * 4 + 2);

  /* no block left: the next fresh block cannot be had, and nothing changes */
  CHECK(pa_alloc_num_free(a) == 0);
  CHECK(pa_alloc_append_slot(a, 0, &slot, &src, &dst) == PA_OK);   /* token 12: offset 3 */
  CHECK(pa_alloc_append_slot(a, 0, &slot, &src, &dst) == PA_ERR_OUT_OF_BLOCKS);
  CHECK(pa_alloc_block_table(a, 0, table, 8, &n, &ntok) == PA_OK && n == 3 && ntok == 12);

  /* freeing the parent releases what only it holds (block 2); 0 and 1 stay shared */
  CHECK(pa_alloc_free_seq(a, 0) == PA_OK);
  CHECK(pa_alloc_refcount(a, 2) == 0 && pa_alloc_refcount(a, 0) == 1);
  CHECK(pa_alloc_num_free(a) == 1);
  CHECK(pa_alloc_free_seq(a, 0) == PA_ERR_NOT_FOUND);
  CHECK(pa_alloc_free_seq(a, 1) == PA_OK);
  CHECK(pa_alloc_num_free(a) == 4);

  CHECK(strcmp(pa_status_string(PA_ERR_OUT_OF_BLOCKS), "no free block left in the pool") == 0);
  pa_alloc_destroy(a);
  printf("ok\n");
  return 0;
}
