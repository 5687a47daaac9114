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

  /* parallel sampling ("深入解析 PagedAttention", 多序列共享): a 34-token prompt in blocks
   * of 4 forked twice; the step's appends copy the shared partial block for two of the
   * three, and the grouping for the shared-prefix decode finds the 32 shared tokens */
  CHECK(pa_alloc_create(32, 4, 0, &a) == PA_OK);
  CHECK(pa_alloc_add_seq(a, 0, 34) == PA_OK);
  CHECK(pa_alloc_fork(a, 0, 1) == PA_OK && pa_alloc_fork(a, 0, 2) == PA_OK);
  const int64_t ids[3] = {0, 1, 2};
  int64_t slots[3];
  int32_t pairs[6];
  int npairs = -1;
  CHECK(pa_alloc_append_slots(a, ids, 3, slots, pairs, &npairs) == PA_OK && npairs == 2);
  int32_t group_of[3], group_prefix[3], group_members[3 * 4];
  int ngroups = -1;
  CHECK(pa_alloc_prefix_groups(a, ids, 3, 4, PA_SHARED_PREFIX_ALIGN, group_of, group_prefix,
                               group_members, &ngroups) == PA_OK);
  CHECK(ngroups == 1 && group_prefix[0] == 32);
  CHECK(group_of[0] == 0 && group_of[1] == 0 && group_of[2] == 0);
  CHECK(group_members[0] == 0 && group_members[1] == 1 && group_members[2] == 2 &&
        group_members[3] == -1);
  pa_alloc_destroy(a);

  /* the step pipeline's input slot: the shared-prefix layout extends the plain one */
  size_t off6[6], off10[10];
  const size_t plain = pa_pipeline_input_bytes(3, 8, 2, 128, 16, PA_BF16, off6);
  const size_t sp = pa_pipeline_input_bytes_prefix(3, 8, 2, 128, 16, PA_BF16, 4, off10);
  CHECK(plain > 0 && sp > plain && off10[6] == plain);
  for (int i = 0; i < 6; ++i) CHECK(off10[i] == off6[i]);
  CHECK(pa_pipeline_input_bytes_prefix(3, 8, 2, 128, 16, PA_BF16, 0, NULL) == plain);
  CHECK(pa_pipeline_input_bytes_prefix(3, 8, 2, 128, 16, PA_BF16, 33, NULL) == 0);
  printf("ok\n");
  return 0;
}
