/* A plain C99 client of libpa.so: compiled with a C compiler against
 * include/pa.h alone, it runs the host-side calls (no GPU needed) and
 * prints what it sees, one "key value..." line each, for
 * tests/test_abi_c_client.py to check.
 *
 * It replays the worked example of "Paged attention in LLMs" (section "A
 * worked example": a 14-token reply in blocks of 5 holds 3 blocks and 15
 * slots), then a fork and the copy-on-write of its shared partial block,
 * an append that does not fit (all-or-nothing), and argument errors that
 * return before any launch. */
#include <stdio.h>
#include <string.h>

#include "pa.h"

static int check(int rc, const char* what) {
  if (rc != PA_OK) printf("error %s %d %s\n", what, rc, pa_last_error_string());
  return rc;
}

int main(void) {
  pa_alloc* a = NULL;
  int64_t slots[32];
  int32_t cow[8][2];
  int32_t table[8];
  int64_t stats[5];
  int ncow = 0, n = 0, nfree = 0, rc, i;

  printf("version %d\n", pa_version());
  if (check(pa_alloc_create(8, 5, NULL, &a), "create")) return 1;
  if (check(pa_alloc_add_seq(a, 7), "add_seq")) return 1;
  if (check(pa_alloc_append(a, 7, 14, slots, &cow[0][0], 8, &ncow), "append")) return 1;
  printf("slots");
  for (i = 0; i < 14; ++i) printf(" %lld", (long long)slots[i]);
  printf("\n");
  if (check(pa_alloc_block_table(a, 7, table, 8, &n), "table")) return 1;
  printf("table");
  for (i = 0; i < n; ++i) printf(" %d", table[i]);
  printf("\n");
  if (check(pa_alloc_stats(a, stats), "stats")) return 1;
  printf("stats %lld %lld %lld %lld %lld\n", (long long)stats[0], (long long)stats[1], (long long)stats[2],
         (long long)stats[3], (long long)stats[4]);

  /* fork, then the child's next token lands in the shared partial block */
  if (check(pa_alloc_fork(a, 7, 8), "fork")) return 1;
  if (check(pa_alloc_refcount(a, table[2], &n), "refcount")) return 1;
  printf("refcount_after_fork %d\n", n);
  if (check(pa_alloc_append(a, 8, 1, slots, &cow[0][0], 8, &ncow), "append_child")) return 1;
  printf("cow %d %d %d slot %lld\n", ncow, cow[0][0], cow[0][1], (long long)slots[0]);
  if (check(pa_alloc_block_table(a, 8, table, 8, &n), "table_child")) return 1;
  printf("child_table");
  for (i = 0; i < n; ++i) printf(" %d", table[i]);
  printf("\n");

  /* an append that does not fit changes nothing */
  pa_alloc_num_free(a, &nfree);
  rc = pa_alloc_append(a, 7, 40, slots, &cow[0][0], 8, &ncow);
  pa_alloc_num_free(a, &n);
  printf("oom %d free_before %d free_after %d\n", rc == PA_ERR_OOM, nfree, n);

  /* argument errors come back before anything is launched */
  rc = pa_reshape_and_cache(NULL, NULL, NULL, NULL, 4, 8, 2, 16, 7, NULL);
  printf("invalid %d %s\n", rc == PA_ERR_INVALID, strstr(pa_last_error_string(), "multiple of 8") ? "msg" : "nomsg");
  rc = pa_decode(NULL, NULL, NULL, NULL, NULL, 0, 8, 2, 128, 16, 10, 4, 0, 1.0f, NULL, 0, NULL);
  printf("empty_decode %d\n", rc == PA_OK);

  pa_alloc_destroy(a);
  printf("done\n");
  return 0;
}
