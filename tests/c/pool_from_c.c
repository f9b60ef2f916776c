/* The host half of the C ABI used from plain C (no Python, no GPU): the block pool walks the worked
 * example of "Nano-vLLM-Ascend: lightweight LLM inference framework for Ascend NPU", section 2.1
 * (1000 tokens in 16-token blocks: 63 blocks, 1008 slots), shares a prefix by reference counts, copies a
 * shared partial block on append, and returns every block when the sequences are freed.
 * Prints "ok" and exits 0, or names the first failed check and exits 1. */
#include <stdio.h>
#include <stdlib.h>

#include "paged_attn.h"

#define CHECK(cond)                                                     \
  do {                                                                  \
    if (!(cond)) {                                                      \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      return 1;                                                         \
    }                                                                   \
  } while (0)

static int invariants(const pa_pool* p) {
  pa_pool_stats_t st;
  if (pa_pool_stats(p, &st) != PA_OK) return 0;
  return st.table_refs == st.ref_sum && st.free_blocks + st.used_blocks == st.num_blocks;
}

int main(void) {
  enum { NB = 200, BS = 16 };
  pa_pool* p = pa_pool_create(NB, BS, NULL);
  CHECK(p != NULL);
  CHECK(pa_pool_create(-1, BS, NULL) == NULL);

  /* 1000 tokens -> 63 blocks, 1008 slots, 8 unused: 0.79 % */
  CHECK(pa_seq_alloc(p, 1, 1000) == PA_OK);
  int len = 0, blocks = 0;
  CHECK(pa_seq_info(p, 1, &len, &blocks) == PA_OK && len == 1000 && blocks == 63);
  pa_pool_stats_t st;
  CHECK(pa_pool_stats(p, &st) == PA_OK && st.used_blocks == 63 && st.free_blocks == NB - 63);
  CHECK(st.utilisation > 0.992 && st.utilisation < 0.993); /* 1000 / 1008 */
  CHECK(pa_seq_alloc(p, 1, 5) == PA_ERR_NOT_FOUND);        /* id already in use */

  /* a child sharing the first 992 tokens (62 full blocks): counts go to 2, nothing is copied */
  CHECK(pa_seq_fork(p, 1, 2, 992) == PA_OK);
  int64_t ids[2] = {1, 2};
  int32_t table[2][64], lens[2];
  CHECK(pa_pool_block_table(p, ids, 2, &table[0][0], 64, lens) == PA_OK);
  CHECK(lens[0] == 1000 && lens[1] == 992 && table[1][62] == -1);
  for (int j = 0; j < 62; ++j) CHECK(table[0][j] == table[1][j] && pa_pool_ref_count(p, table[0][j]) == 2);
  CHECK(pa_pool_ref_count(p, table[0][62]) == 1);
  CHECK(invariants(p));

  /* the child appends into a fresh block (its 62 blocks are full): no copy */
  int64_t slot = -7;
  int32_t cow[2] = {-1, -1};
  int ncow = -1;
  CHECK(pa_seq_append(p, 2, 1, &slot, cow, &ncow) == PA_OK && ncow == 0);
  CHECK(pa_pool_block_table(p, ids, 2, &table[0][0], 64, lens) == PA_OK);
  CHECK(slot == (int64_t)table[1][62] * BS + 0 && table[1][62] != table[0][62]);

  /* a second child sharing all 1000 tokens, including the partly filled last block; appending to it
   * copies that block first (copy-on-write) and writes into the copy */
  CHECK(pa_seq_fork(p, 1, 3, 1000) == PA_OK);
  const int32_t last_shared = table[0][62];
  CHECK(pa_pool_ref_count(p, last_shared) == 2);
  CHECK(pa_seq_append(p, 3, 1, &slot, cow, &ncow) == PA_OK && ncow == 1);
  CHECK(cow[0] == last_shared && cow[1] != last_shared);
  CHECK(slot == (int64_t)cow[1] * BS + 1000 % BS);
  CHECK(pa_pool_ref_count(p, last_shared) == 1 && pa_pool_ref_count(p, cow[1]) == 1);
  CHECK(invariants(p));

  /* one call for a whole batch: sequences 1 and 2 gain two tokens each, in order */
  {
    int64_t bids[2] = {1, 2}, bslots[4];
    int32_t bcounts[2] = {2, 2}, bpairs[4];
    int bncow = -1;
    CHECK(pa_pool_append_batch(p, bids, bcounts, 2, bslots, bpairs, &bncow) == PA_OK && bncow == 0);
    CHECK(pa_pool_block_table(p, ids, 2, &table[0][0], 64, lens) == PA_OK && lens[0] == 1002 && lens[1] == 995);
    CHECK(bslots[0] == (int64_t)table[0][62] * BS + 1000 % BS && bslots[1] == bslots[0] + 1);
    CHECK(bslots[2] == (int64_t)table[1][62] * BS + 1 && bslots[3] == bslots[2] + 1);
    int64_t dup[2] = {1, 1};
    CHECK(pa_pool_append_batch(p, dup, bcounts, 2, NULL, NULL, NULL) == PA_ERR_INVALID);
  }

  /* too many tokens: refused, pool unchanged */
  CHECK(pa_pool_stats(p, &st) == PA_OK);
  const int64_t free_before = st.free_blocks;
  CHECK(pa_seq_alloc(p, 9, (int)((free_before + 1) * BS)) == PA_ERR_OOM);
  CHECK(pa_pool_stats(p, &st) == PA_OK && st.free_blocks == free_before && st.num_seqs == 3);

  /* freeing every sequence returns every block */
  CHECK(pa_seq_free(p, 1) == PA_OK && pa_seq_free(p, 2) == PA_OK && pa_seq_free(p, 3) == PA_OK);
  CHECK(pa_seq_free(p, 3) == PA_ERR_NOT_FOUND);
  CHECK(pa_pool_stats(p, &st) == PA_OK && st.free_blocks == NB && st.used_blocks == 0 && st.ref_sum == 0);
  pa_pool_destroy(p);

  /* device calls validate on the host and launch nothing when an argument is wrong */
  CHECK(pa_write_kv(NULL, NULL, NULL, 4, NULL, NULL, 8, BS, 2, 64, PA_BF16, NULL) == PA_ERR_INVALID);
  CHECK(pa_write_kv(NULL, NULL, NULL, 0, (void*)0x10000, (void*)0x10000, 8, 24, 2, 64, PA_BF16, NULL) ==
        PA_ERR_UNSUPPORTED);
  CHECK(pa_write_kv(NULL, NULL, NULL, 0, (void*)0x10000, (void*)0x10000, 8, BS, 2, 64, PA_BF16, NULL) == PA_OK);
  CHECK(pa_strerror(PA_ERR_OOM) != NULL && pa_version() != NULL);
  printf("ok\n");
  return 0;
}
