/* A plain C11 caller of libpa.so: the boundary is a C ABI.  It drives a
 * host-only pool (no GPU) through reservation, fork, prefix reuse (the
 * 103-token prompt that reuses 96 tokens with 16-token blocks,
 * kv-cache-pagedattention-serving, Beyond paging: radix trees and continuous
 * batching), the cached list, a host state checkpoint and restore, swap
 * sizing and error reporting, and prints "ok" when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "pa.h"

static int failures = 0;
#define EXPECT(c)                                                  \
  do {                                                             \
    if (!(c)) {                                                    \
      fprintf(stderr, "line %d: %s (%s)\n", __LINE__, #c, pa_last_error()); \
      ++failures;                                                  \
    }                                                              \
  } while (0)

int main(void) {
  pa_pool_desc d;
  memset(&d, 0, sizeof d);
  d.num_layers = 80;
  d.num_kv_heads = 8;
  d.head_dim = 128;
  d.block_size = 16;
  d.num_blocks = 64;
  d.max_seqs = 4;
  d.max_blocks_per_seq = 16;
  d.kv_dtype = PA_BF16;
  d.act_dtype = PA_BF16;
  pa_pool *p = NULL;
  EXPECT(pa_pool_create(&d, &p) == PA_OK && p != NULL);
  if (!p) return 1;

  int32_t tokens[103];
  for (int i = 0; i < 103; ++i) tokens[i] = 1000 + 7 * i;
  int32_t cached = -1;
  EXPECT(pa_alloc_blocks_prefix(p, 0, 103, tokens, &cached) == PA_OK && cached == 0);
  EXPECT(pa_prefix_register(p, 0, 103, tokens) == PA_OK);
  EXPECT(pa_prefix_match(p, 103, tokens, &cached) == PA_OK && cached == 96);
  EXPECT(pa_alloc_blocks_prefix(p, 1, 103, tokens, &cached) == PA_OK && cached == 96);

  int32_t len = 0, nblocks = 0, t0[16], t1[16];
  EXPECT(pa_get_seq(p, 0, &len, t0, 16, &nblocks) == PA_OK && len == 103 && nblocks == 7);
  EXPECT(pa_get_seq(p, 1, &len, t1, 16, &nblocks) == PA_OK && nblocks == 7);
  EXPECT(memcmp(t0, t1, 6 * sizeof(int32_t)) == 0 && t0[6] != t1[6]);

  int32_t refs[64];
  EXPECT(pa_get_refcounts(p, refs, 64) == PA_OK && refs[t0[0]] == 2 && refs[t0[6]] == 1);
  EXPECT(pa_fork_cow(p, 1, 2) == PA_OK);
  EXPECT(pa_alloc_blocks(p, 2, 104, NULL) == PA_OK); /* copy-on-write of the shared tail */
  int32_t cow[8], ncow = 0;
  EXPECT(pa_get_cow_log(p, cow, 4, &ncow) == PA_OK && ncow == 1 && cow[0] == t1[6]);

  EXPECT(pa_free(p, 0) == PA_OK && pa_free(p, 1) == PA_OK && pa_free(p, 2) == PA_OK);
  int32_t idle[64], nidle = 0;
  EXPECT(pa_get_cached_blocks(p, idle, 64, &nidle) == PA_OK && nidle == 6);
  EXPECT(idle[0] == t0[5] && idle[5] == t0[0]); /* longer prefixes leave first */

  /* host state checkpoint: save, change, restore */
  size_t img = 0, wrote = 0;
  EXPECT(pa_state_size(p, &img) == PA_OK && img > 0 && img % 4 == 0);
  void *buf = malloc(img);
  EXPECT(buf != NULL);
  if (!buf) return 1;
  EXPECT(pa_state_save(p, buf, img - 4, &wrote) == PA_ERR_INVALID_ARG); /* too small */
  EXPECT(pa_state_save(p, buf, img, &wrote) == PA_OK && wrote == img);
  int32_t free_before[64], nfree_before = 0, free_after[64], nfree_after = 0;
  EXPECT(pa_get_free_list(p, free_before, 64, &nfree_before) == PA_OK);
  EXPECT(pa_alloc_blocks(p, 3, 200, NULL) == PA_OK); /* 13 blocks */
  EXPECT(pa_state_load(p, buf, img - 4) == PA_ERR_INVALID_ARG); /* truncated: nothing changes */
  EXPECT(pa_get_seq(p, 3, &len, t0, 16, &nblocks) == PA_OK && len == 200);
  EXPECT(pa_state_load(p, buf, img) == PA_OK);
  EXPECT(pa_get_seq(p, 3, &len, t0, 16, &nblocks) == PA_ERR_NO_SEQ);
  EXPECT(pa_get_free_list(p, free_after, 64, &nfree_after) == PA_OK && nfree_after == nfree_before &&
         memcmp(free_before, free_after, sizeof(int32_t) * (size_t)nfree_before) == 0);
  EXPECT(pa_get_cached_blocks(p, idle, 64, &nidle) == PA_OK && nidle == 6);
  free(buf);

  size_t bytes = 0;
  EXPECT(pa_swap_bytes(p, 1525, &bytes) == PA_OK && bytes == (size_t)503316480);
  EXPECT(pa_swap_out(p, 0, NULL, 0, NULL) == PA_ERR_INVALID_ARG); /* host-only pool */
  EXPECT(pa_fork_cow(p, 3, 0) == PA_ERR_NO_SEQ);
  EXPECT(strlen(pa_last_error()) > 0);
  EXPECT(strcmp(pa_status_string(PA_ERR_NO_SEQ), "PA_ERR_NO_SEQ") == 0);
  pa_pool_destroy(p);
  if (failures) return 1;
  printf("ok\n");
  return 0;
}
