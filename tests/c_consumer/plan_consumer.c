/* A plain C consumer of libbat.so (no Python, no CUDA headers): builds host-only plans
 * through the C ABI of include/bat.h, checks their summaries and the error codes of bad
 * calls, and prints one line of results for the test that compiles and runs it. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "bat.h"

static int failures = 0;
#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

int main(void) {
  CHECK((bat_version() >> 16) == 1);

  /* Three requests: two read prefix 0 (17 rows), one reads none; suffixes of 5, 4 and 191 rows. */
  const int32_t req_prefix[3] = {0, -1, 0};
  const int64_t suffix_offsets[4] = {0, 5, 9, 200};
  const int64_t prefix_offsets[2] = {0, 17};
  bat_plan_options opts;
  memset(&opts, 0, sizeof(opts));
  opts.host_only = 1;
  opts.num_sms = 148;

  bat_plan* plan = NULL;
  CHECK(bat_plan_create(req_prefix, suffix_offsets, prefix_offsets, 3, 1, 4, 128, BAT_BF16, &opts, NULL, &plan) ==
        BAT_OK);
  CHECK(plan != NULL);
  bat_plan_info_t info;
  memset(&info, 0, sizeof(info));
  CHECK(bat_plan_info(plan, &info) == BAT_OK);
  CHECK(info.R == 3 && info.P == 1 && info.H == 4 && info.d == 128 && info.on_device == 0);
  CHECK(info.T_suf == 200 && info.T_cache == 17);
  /* Query tiles: 1 + 1 + 2 = 4 per head; each item holds at most two of them. */
  CHECK(info.n_items >= 2 * 4 && info.n_items <= 4 * 4);

  /* The work list copy: 64-byte records; too small a buffer is rejected. */
  const size_t bytes = (size_t)info.n_items * 64;
  unsigned char* items = (unsigned char*)malloc(bytes);
  CHECK(items != NULL);
  CHECK(bat_plan_items(plan, items, bytes - 1) == BAT_ERR_INVALID_ARG);
  CHECK(bat_plan_items(plan, items, bytes) == BAT_OK);
  /* First field of every record is the head: each head appears n_items / H times. */
  int64_t per_head[4] = {0, 0, 0, 0};
  for (int64_t i = 0; i < info.n_items; ++i) {
    int32_t head;
    memcpy(&head, items + i * 64, sizeof(head));
    CHECK(head >= 0 && head < 4);
    if (head >= 0 && head < 4) per_head[head]++;
  }
  CHECK(per_head[0] == per_head[1] && per_head[1] == per_head[2] && per_head[2] == per_head[3]);
  free(items);
  CHECK(bat_plan_destroy(plan) == BAT_OK);
  CHECK(bat_plan_destroy(NULL) == BAT_OK);

  /* Prefix-side plan: two prefixes of 17 and 300 rows; no request reads a cached prefix. */
  const int64_t src_offsets[3] = {0, 17, 317};
  plan = NULL;
  CHECK(bat_plan_create_prefix_side(src_offsets, 2, 2, 64, BAT_BF16, &opts, NULL, &plan) == BAT_OK);
  CHECK(bat_plan_info(plan, &info) == BAT_OK);
  CHECK(info.R == 2 && info.P == 0 && info.T_suf == 317 && info.T_cache == 0);
  CHECK(bat_plan_destroy(plan) == BAT_OK);

  /* Errors come back as codes with a message, never as a crash. */
  plan = NULL;
  CHECK(bat_plan_create(req_prefix, suffix_offsets, prefix_offsets, 3, 1, 0, 128, BAT_BF16, &opts, NULL, &plan) ==
        BAT_ERR_INVALID_ARG);
  CHECK(plan == NULL);
  CHECK(strlen(bat_last_error()) > 0);
  CHECK(bat_plan_create(req_prefix, suffix_offsets, prefix_offsets, 3, 1, 2, 32, BAT_BF16, &opts, NULL, &plan) ==
        BAT_ERR_UNSUPPORTED);
  const int32_t bad_prefix[3] = {0, 5, 0};
  CHECK(bat_plan_create(bad_prefix, suffix_offsets, prefix_offsets, 3, 1, 2, 128, BAT_BF16, &opts, NULL, &plan) ==
        BAT_ERR_INVALID_ARG);
  CHECK(bat_plan_info(NULL, &info) == BAT_ERR_INVALID_ARG);

  printf("c consumer: %s (%d failed checks)\n", failures ? "FAIL" : "ok", failures);
  return failures ? 1 : 0;
}
