/* A plain C99 client of the library's C ABI (include/mla.h), built and run by the CPU
 * test suite: it plans a small step on the host only (no CUDA call is made), inspects
 * the plan, re-plans it with unchanged and changed tables, and checks the documented
 * error codes.  It prints one "key value" line per check for the test to read. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "mla.h"

int main(void) {
  mla_dims d;
  mla_plan_options o;
  mla_plan_info info;
  mla_plan_t p = NULL;
  mla_status st;
  /* two rows: 1 query over 37 keys, 3 queries over 150 keys; 16 heads, pages of 16 */
  const int32_t qo[3] = {0, 1, 4};
  const int32_t kvp[3] = {0, 3, 13};
  const int32_t kvi[13] = {4, 9, 1, 0, 2, 3, 5, 6, 7, 8, 10, 11, 12};
  const int32_t last[2] = {5, 6};
  int32_t kv_len[2] = {0, 0};
  int32_t reused = -1;
  int32_t kvi2[13];

  d.num_heads = 16;
  d.kv_lora_rank = 512;
  d.rope_dim = 64;
  d.page_size = 16;
  d.num_pages = 16;
  d.sm_scale = 0.0721687836f;
  memset(&o, 0, sizeof(o));
  o.host_only = 1;

  printf("supports %d %d %d\n", mla_supports(512, 64, 16, 16), mla_supports(512, 0, 128, 64),
         mla_supports(512, 32, 16, 16));
  st = mla_plan(&d, 2, qo, kvp, kvi, last, 1, NULL, &o, &p);
  printf("plan %d %s\n", (int)st, mla_status_string(st));
  if (st != MLA_OK) return 1;
  st = mla_plan_get_info(p, &info);
  printf("info %d batch %d tokens %d work %d merge %d\n", (int)st, info.batch, info.total_tokens, info.num_work,
         info.num_merge);
  st = mla_plan_describe(p, kv_len, NULL, NULL, NULL);
  printf("kv_len %d %d %d\n", (int)st, kv_len[0], kv_len[1]);
  st = mla_plan_update(p, 2, qo, kvp, kvi, last, NULL, &reused);
  printf("update_same %d %d\n", (int)st, reused);
  memcpy(kvi2, kvi, sizeof(kvi));
  kvi2[0] = 15;
  st = mla_plan_update(p, 2, qo, kvp, kvi2, last, NULL, &reused);
  printf("update_changed %d %d\n", (int)st, reused);
  kvi2[0] = 16; /* out of range: rejected, the plan keeps its step */
  st = mla_plan_update(p, 2, qo, kvp, kvi2, last, NULL, &reused);
  printf("update_bad %d\n", (int)st);
  st = mla_run(p, NULL, NULL, NULL, NULL, NULL, NULL); /* a host-only plan cannot run */
  printf("run_host_only %d\n", (int)st);
  st = mla_merge_state(NULL, NULL, NULL, NULL, NULL, NULL, -1, NULL);
  printf("merge_state_bad %d\n", (int)st);
  mla_plan_destroy(p);
  mla_plan_destroy(NULL);
  printf("done\n");
  return 0;
}
