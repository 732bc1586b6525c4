/* The C ABI from plain C: moe.h compiles as C99, libmoe.so links, and the
 * calls that need no GPU behave as declared (version, status strings, the
 * host-side expert-parallel plan, argument validation before any launch).
 * Built and run by tests/test_abi.py. Prints "ok" and returns 0 on success. */
#include <stdio.h>
#include <string.h>

#include "moe.h"

#define CHECK(c)                                             \
  do {                                                       \
    if (!(c)) {                                              \
      fprintf(stderr, "failed: %s (line %d)\n", #c, __LINE__); \
      return 1;                                              \
    }                                                        \
  } while (0)

int main(void) {
  CHECK(moe_version() >= 100);
  CHECK(strcmp(moe_strerror(MOE_OK), moe_strerror(MOE_ERR_INVALID_ARG)) != 0);
  CHECK(strcmp(moe_strerror(-99), "unknown status") == 0);

  /* two ranks, two experts each; this rank routes {1, 2 | 3, 0} rows and
   * receives {1, 2} from rank 0 and {3, 0} from rank 1 */
  const int32_t local[4] = {1, 2, 3, 0};
  const int32_t recv[4] = {1, 2, 3, 0};
  long long send_splits[2], recv_splits[2], n_recv = -1;
  int32_t offsets[3], regroup[6], ungroup[6];
  CHECK(moe_ep_plan(local, recv, 2, 2, 6, send_splits, recv_splits, offsets, regroup, ungroup,
                    &n_recv) == MOE_OK);
  CHECK(n_recv == 6);
  CHECK(send_splits[0] == 3 && send_splits[1] == 3);
  CHECK(recv_splits[0] == 3 && recv_splits[1] == 3);
  /* expert 0: rank 0's row 0, rank 1's rows 3..5; expert 1: rank 0's rows 1..2 */
  CHECK(offsets[0] == 0 && offsets[1] == 4 && offsets[2] == 6);
  {
    const int32_t want[6] = {0, 3, 4, 5, 1, 2};
    int i;
    for (i = 0; i < 6; ++i) CHECK(regroup[i] == want[i]);
    for (i = 0; i < 6; ++i) CHECK(ungroup[regroup[i]] == i);
  }
  /* too little capacity: an error and nothing written */
  n_recv = -1;
  CHECK(moe_ep_plan(local, recv, 2, 2, 5, send_splits, recv_splits, offsets, regroup, ungroup,
                    &n_recv) == MOE_ERR_INVALID_ARG);
  CHECK(n_recv == -1);

  /* validation happens on the host before CUDA is touched */
  CHECK(moe_route(NULL, NULL, NULL, 64, 256, 16, 4, MOE_GATE_SIGMOID_BIAS, 1.0f, NULL, NULL,
                  NULL, NULL) == MOE_ERR_INVALID_ARG);
  CHECK(moe_combine(NULL, NULL, NULL, NULL, NULL, -1, 256, 4, NULL, NULL) == MOE_ERR_INVALID_ARG);
  CHECK(moe_gather_rows(NULL, 4, NULL, 4, 12, NULL, NULL) == MOE_ERR_UNSUPPORTED_SHAPE);

  printf("ok\n");
  return 0;
}
