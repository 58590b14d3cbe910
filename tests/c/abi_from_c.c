/*
 * The C ABI used from plain C99: include/mep.h needs no CUDA or C++ header,
 * and the host-side calls behave as the header states.  Built and run by
 * tests/test_abi_cpu.py with gcc; no GPU is touched (every call below is
 * rejected or answered before any CUDA call).
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "mep.h"

#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      fprintf(stderr, "FAILED line %d: %s\n", __LINE__, #cond);  \
      return 1;                                                  \
    }                                                            \
  } while (0)

int main(void) {
  mep_shape_t s = {8, 4096, 64, 6};
  mep_shape_t bad = {3, 4, 64, 6}; /* E % R != 0 */
  mep_plan_t plan;
  int32_t idx_dummy[4];
  uint16_t rows[64];
  mep_ipc_handle_t h;
  void *p = NULL;

  CHECK(mep_version() == MEP_VERSION);
  CHECK(strcmp(mep_status_string(MEP_OK), "ok") == 0);
  CHECK(mep_status_string(MEP_ERR_TIMEOUT) != NULL);
  CHECK(mep_plan_workspace_bytes(s) > 0);
  CHECK(mep_plan_workspace_bytes(bad) == 0);

  memset(&plan, 0, sizeof plan);
  /* NULL plan fields and NULL inputs are host-side errors */
  CHECK(mep_plan(s, idx_dummy, &plan, NULL, 0, NULL) != MEP_OK);
  CHECK(mep_dispatch(s, 2048, NULL, rows, rows, NULL) == MEP_ERR_INVALID_ARG);
  CHECK(mep_combine(bad, 2048, &plan, rows, NULL, rows, NULL) == MEP_ERR_INVALID_ARG);
  CHECK(mep_reduce_replica_grads(s, &plan, 0, NULL, NULL, NULL) == MEP_OK); /* P = 0: no-op */
  CHECK(mep_dispatch_ranked_tokens(s, 2048, &plan, -1, 1, rows, NULL, NULL) == MEP_ERR_INVALID_ARG);
  CHECK(mep_reduce_replica_grads_ranked(s, &plan, 16, s.R, NULL, 1, NULL, NULL) ==
        MEP_ERR_INVALID_ARG);
  CHECK(mep_ipc_export(NULL, 16, &h) == MEP_ERR_INVALID_ARG);
  CHECK(mep_ipc_open(NULL, &p) == MEP_ERR_INVALID_ARG);
  CHECK(sizeof(mep_segment_t) == 16);
  CHECK(sizeof(mep_ipc_handle_t) == 80);

  mep_set_wait_limit_ns(250000000ull);
  CHECK(mep_get_wait_limit_ns() == 250000000ull);
  mep_set_wait_limit_ns(1000000000ull);
  puts("c abi ok");
  return 0;
}
