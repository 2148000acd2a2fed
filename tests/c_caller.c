/*
 * A plain C99 caller of libretention: includes only include/retention.h and
 * links the shared library, with no C++ or torch in between.  It makes only
 * calls that return before any launch (argument validation, queries, status
 * names), so it runs without a GPU.  Used by tests/test_abi.py.
 */
#include <stdint.h>
#include <stdio.h>

#include "retention.h"

#define CHECK(cond)                                           \
  do {                                                        \
    if (!(cond)) {                                            \
      printf("FAIL line %d: %s\n", __LINE__, #cond);          \
      return 1;                                               \
    }                                                         \
  } while (0)

int main(void) {
  void* fake = (void*)(uintptr_t)0x10000; /* never dereferenced: validation fails first */
  float gamma[2] = {0.5f, 0.9f};
  float bad_gamma[2] = {0.5f, 1.5f};
  ret_shape s = {1, 2, 64, 64, 128};
  char buf[32];

  CHECK(retention_abi_version() >= 100);
  CHECK(retention_status_str(RET_OK) != NULL);
  CHECK(retention_status_str(RET_ETIMEOUT) != NULL);
  /* invalid decays and a null output are rejected before anything launches */
  CHECK(retention_parallel(fake, fake, fake, bad_gamma, fake, s, RET_BF16, NULL) == RET_EINVAL);
  CHECK(retention_chunkwise(fake, fake, fake, gamma, NULL, NULL, NULL, 64, s, RET_BF16, NULL, 0, NULL) ==
        RET_EINVAL);
  CHECK(retention_chunkwise(fake, fake, fake, gamma, fake, NULL, NULL, 0, s, RET_BF16, NULL, 0, NULL) ==
        RET_EINVAL);
  CHECK(retention_recurrent_step(fake, fake, fake, gamma, fake, NULL, s, RET_F32, NULL) == RET_EINVAL);
  CHECK(retention_groupnorm_gated(fake, fake, fake, 1e-5f, NULL, NULL, 7, s, RET_BF16, NULL) == RET_EINVAL);
  CHECK(retention_state_fold(fake, NULL, 1, gamma, NULL, fake, s, NULL) == RET_EINVAL);
  /* queries */
  CHECK(retention_chunkwise_backward_state_workspace_bytes(64, s, RET_F32) >
        retention_chunkwise_backward_workspace_bytes(64, s, RET_F32));
  CHECK(retention_chunkwise_state_workspace_bytes(64, s, RET_F32) == 0);
  snprintf(buf, sizeof buf, "%s", retention_status_str(RET_EUNSUPPORTED));
  printf("ok %s\n", buf);
  return 0;
}
