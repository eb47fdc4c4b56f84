/* Plain C99 use of the library's host entry points (no GPU needed): the
 * allocator, the continuous-batching step and its packed form.  Prints one
 * line per check and exits non-zero on the first failure. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "pagedkv.h"

#define CHECK(cond, msg)                                   \
  do {                                                     \
    if (!(cond)) {                                         \
      fprintf(stderr, "FAIL %s: %s\n", msg, kv_last_error()); \
      return 1;                                            \
    }                                                      \
    printf("ok %s\n", msg);                                \
  } while (0)

int main(void) {
  kv_alloc* a = NULL;
  kv_sched* s = NULL;
  CHECK(kv_version() == 1, "version");
  CHECK(kv_alloc_create(64, 16, NULL, &a) == KV_OK, "allocator");
  CHECK(kv_sched_create(a, 8, -1, &s) == KV_OK, "scheduler");
  CHECK(kv_sched_add_request(s, 7, 40) == KV_OK && kv_sched_add_request(s, 8, 16) == KV_OK, "requests");

  const size_t cap = kv_step_packed_bytes(8, 128, 8, 0);
  unsigned char* raw = (unsigned char*)malloc(cap + 16);
  unsigned char* buf = raw + ((16 - ((uintptr_t)raw % 16)) % 16);
  int64_t running[8];
  kv_step_layout lay;
  memset(&lay, 0, sizeof lay);
  CHECK(kv_sched_step_packed(s, NULL, 0, KV_ORDER_LONGEST, 8, buf, cap, running, &lay) == KV_OK, "packed step");
  CHECK(lay.info.batch == 2 && lay.info.num_admitted == 2 && running[0] == 7 && running[1] == 8, "admitted");
  /* 40 + 16 prompt slots, then one appended slot per sequence */
  CHECK(lay.info.num_tokens == 58 && lay.prefill_tokens == 56 && lay.max_prefill_len == 40, "token counts");
  const int32_t* lens = (const int32_t*)(buf + lay.context_lens);
  const int32_t* order = (const int32_t*)(buf + lay.seq_order);
  const int32_t* cu = (const int32_t*)(buf + lay.cu_seqlens);
  CHECK(lens[0] == 41 && lens[1] == 17 && lay.max_context_len == 41, "context lengths");
  CHECK(order[0] == 0 && order[1] == 1 && cu[0] == 0 && cu[1] == 40 && cu[2] == 56, "order and prefill rows");
  /* the packed tables equal kv_sched_outputs' rows at the same width */
  int32_t tables[2 * 8];
  CHECK(kv_sched_outputs(s, NULL, tables, lay.table_width, NULL, NULL, NULL, NULL) == KV_OK, "outputs");
  CHECK(memcmp(tables, buf + lay.block_tables, sizeof(int32_t) * 2 * lay.table_width) == 0, "packed tables");
  const int64_t* slots = (const int64_t*)(buf + lay.slot_mapping);
  int32_t t7[8];
  int n7 = 0;
  CHECK(kv_alloc_block_table(a, 7, t7, 8, &n7) == KV_OK && n7 == 3, "table of sequence 7");
  CHECK(slots[0] == (int64_t)t7[0] * 16 && slots[56] == (int64_t)t7[2] * 16 + 8, "slot mapping");

  const int64_t done = 8;
  CHECK(kv_sched_step_packed(s, &done, 1, KV_ORDER_BATCH, 8, buf, cap, running, &lay) == KV_OK, "finish one");
  CHECK(lay.info.batch == 1 && running[0] == 7 && lay.seq_order == -1 && lay.cu_seqlens == -1, "after finish");
  CHECK(kv_sched_step_packed(s, &done, 1, KV_ORDER_BATCH, 8, buf, cap, running, &lay) == KV_ERR_STATE,
        "unknown finished id rejected");
  free(raw);
  CHECK(kv_sched_destroy(s) == KV_OK && kv_alloc_destroy(a) == KV_OK, "destroy");
  return 0;
}
