/* A plain C99 client of the C ABI: includes both headers, links libpkv.so and
 * uses the calls that need no GPU (status text, version, build kind, the
 * host-side argument checks of the device calls, and the block manager for a
 * prompt, a fork with copy-on-write and a decode step).  Exit status 0 when
 * every result is the documented one. */
#include <stdio.h>
#include <string.h>

#include "pkv.h"
#include "pkv_block_manager.h"

#define CHECK(c)                                                   \
  do {                                                             \
    if (!(c)) {                                                    \
      fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #c); \
      return 1;                                                    \
    }                                                              \
  } while (0)

int main(void) {
  pkv_cache_desc desc;
  pkv_block_manager *bm = NULL;
  int64_t slots[40], pairs[4], ids[2];
  int32_t tables[2 * 8], lens[2], ncopies = -1;

  CHECK(strcmp(pkv_status_string(PKV_OK), "ok") == 0);
  CHECK(pkv_version() >= 100);
  CHECK(pkv_check_build() == 0 || pkv_check_build() == 1);

  desc.num_blocks = 16;
  desc.block_size = 16;
  desc.num_kv_heads = 4;
  desc.head_dim = 64;
  desc.dtype = PKV_F16;
  /* host-side checks return before any device work */
  CHECK(pkv_reshape_and_cache(NULL, NULL, 0, 0, NULL, NULL, desc, NULL, 1, NULL, NULL) == PKV_ERR_NULL_POINTER);
  CHECK(pkv_reshape_and_cache(NULL, NULL, 0, 0, NULL, NULL, desc, NULL, 0, NULL, NULL) == PKV_OK);
  desc.block_size = 12;
  CHECK(pkv_copy_blocks(NULL, NULL, desc, NULL, 1, NULL, NULL) == PKV_ERR_BAD_SHAPE);

  /* block manager: 8 blocks of 16 tokens, tables of 8 entries */
  CHECK(pkv_bm_create(8, 16, 8, &bm) == PKV_OK);
  CHECK(pkv_bm_add_sequence(bm, 7, 20, slots) == PKV_OK);      /* blocks 0, 1 */
  CHECK(slots[0] == 0 && slots[15] == 15 && slots[16] == 16 && slots[19] == 19);
  CHECK(pkv_bm_fork(bm, 7, 8) == PKV_OK);                      /* shares 0, 1 */
  CHECK(pkv_bm_ref_count(bm, 1) == 2);
  ids[0] = 8;
  CHECK(pkv_bm_append(bm, ids, 1, slots, pairs, 1, &ncopies) == PKV_OK);
  CHECK(ncopies == 1 && pairs[0] == 1 && pairs[1] == 2);       /* copy-on-write of block 1 into 2 */
  CHECK(slots[0] == 2 * 16 + 4);                               /* token 20 of request 8 */
  ids[1] = 7;
  CHECK(pkv_bm_block_tables(bm, ids, 2, tables, 8, lens) == PKV_OK);
  CHECK(lens[0] == 21 && lens[1] == 20);
  CHECK(tables[0] == 0 && tables[1] == 2 && tables[2] == -1);
  CHECK(tables[8] == 0 && tables[9] == 1);
  CHECK(pkv_bm_free_sequence(bm, 7) == PKV_OK && pkv_bm_ref_count(bm, 1) == 0);
  CHECK(pkv_bm_num_free_blocks(bm) == 6);
  pkv_bm_destroy(bm);
  printf("c client ok\n");
  return 0;
}
