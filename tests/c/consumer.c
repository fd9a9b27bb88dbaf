/* A plain C99 consumer of the library: compiles against include/fg.h alone
 * and calls the entry points that need no GPU (status strings, the rotary
 * table, the host-side work plan, argument errors). Built and run by
 * tests/test_c_consumer.py. */
#include <stdio.h>
#include <string.h>

#include "fg.h"

static int fails = 0;
#define CHECK(cond)                                                  \
  do {                                                               \
    if (!(cond)) {                                                   \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      ++fails;                                                       \
    }                                                                \
  } while (0)

int main(void) {
  float c[2 * 4], s[2 * 4];
  int32_t ql[3] = {300, 1, 1}, cl[3] = {0, 4000, 700};
  int64_t counts[12];
  fg_ragged_batch* b = NULL;

  CHECK(strcmp(fg_status_string(FG_OK), "FG_OK") == 0);
  /* position 0 is the identity rotation: cos 1, sin 0 */
  CHECK(fg_rotary_table(10000.0, 8, 0, 2, c, s) == FG_OK);
  CHECK(c[0] == 1.0f && s[0] == 0.0f && c[3] == 1.0f);
  CHECK(fg_rotary_table(10000.0, 7, 0, 1, c, s) == FG_ERR_INVALID_ARG);
  /* the plan of a prefill chunk and two decodes, MHA d = 128 */
  CHECK(fg_plan_describe(ql, cl, 3, 4, 1, 128, 0, 1, 148, NULL, 0, counts) == FG_OK);
  CHECK(counts[2] == 2 * 4);        /* 300 tokens = two 256-row units per kv head */
  CHECK(counts[3] >= 2 * 4);        /* the decodes, split on the tensor-core decode path */
  CHECK(counts[11] % 256 == 0);
  CHECK(fg_plan_describe(ql, cl, 3, 4, 1, 96, 0, 1, 148, NULL, 0, counts) == FG_ERR_INVALID_ARG);
  /* a batch handle allocates nothing until its first put */
  CHECK(fg_ragged_batch_create(64, 4, 8, &b) == FG_OK && b != NULL);
  CHECK(fg_ragged_batch_put(b, NULL, 0, NULL, NULL, NULL, NULL, 1, NULL) == FG_ERR_INVALID_ARG);
  CHECK(fg_ragged_batch_destroy(b) == FG_OK);
  CHECK(fg_ragged_batch_destroy(NULL) == FG_OK);
  if (fails) return 1;
  printf("ok\n");
  return 0;
}
