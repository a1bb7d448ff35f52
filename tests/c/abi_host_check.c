/* A C99 caller of the kd C ABI.  Only calls that fail host-side validation
 * (and so launch nothing) or need no device are made, so it runs without a
 * GPU.  Exit status 0 means every check held. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "kd.h"

static int failures = 0;

static void expect(int cond, const char* what) {
  if (!cond) {
    fprintf(stderr, "FAILED: %s\n", what);
    ++failures;
  }
}

int main(void) {
  /* a 1024-aligned address that is never dereferenced */
  void* const fake = (void*)(uintptr_t)0x7F0000000000ull;
  const size_t huge = (size_t)1 << 40;

  expect(kd_version() >> 16 == 1, "major version 1");
  expect(strcmp(kd_status_string(KD_OK), "KD_OK") == 0, "status string of KD_OK");
  expect(strcmp(kd_status_string(KD_ERR_BAD_INDEX), "KD_ERR_BAD_INDEX") == 0,
         "status string of KD_ERR_BAD_INDEX");

  expect(kd_fused_kl_workspace_size(32768, 4096, 131072, 100, 2048, KD_DTYPE_BF16) > 0,
         "workspace size of the 32K head");
  expect(kd_fused_kl_workspace_size(0, 8, 8, 1, 1, KD_DTYPE_BF16) == 0, "workspace size of T=0");
  expect(kd_topk_workspace_size(8192, 131072, 100) >= 4, "top-K workspace size");

  expect(kd_fused_kl_fwd(NULL, fake, KD_DTYPE_BF16, 256, 256, 4096, fake, fake, 16, 64, 1.0f,
                         fake, fake, NULL, fake, huge, NULL) == KD_ERR_INVALID_ARG,
         "forward rejects a null h");
  expect(kd_fused_kl_bwd(fake, fake, KD_DTYPE_BF16, 256, 12, 4096, fake, fake, 16, 64, 1.0f,
                         fake, NULL, fake, fake, 0, fake, huge, NULL) == KD_ERR_UNSUPPORTED,
         "backward rejects d % 8 != 0");
  expect(kd_fused_kl_fwd_ex(fake, fake, KD_DTYPE_BF16, 256, 256, 4096, fake, fake, 16, 64, 1.0f,
                            0x4u, fake, fake, NULL, fake, huge, NULL) == KD_ERR_INVALID_ARG,
         "forward rejects unknown flags");
  expect(kd_fused_kl_bwd_ex(fake, fake, KD_DTYPE_BF16, 256, 256, 4096, fake, fake, 16, 64, 0.0f,
                            KD_KL_LOGPROB_CACHE | KD_KL_TAU_SQUARED, fake, NULL, fake, fake, 0,
                            fake, huge, NULL) == KD_ERR_INVALID_ARG,
         "backward rejects tau = 0");
  expect(kd_topk_build(fake, KD_DTYPE_BF16, 8, 100, 101, fake, fake, fake, huge, NULL) ==
             KD_ERR_INVALID_ARG,
         "top-K rejects K > V");
  expect(kd_set_wait_limit_ns(10) == KD_ERR_INVALID_ARG, "wait limit below 1000 ns");
  expect(kd_read_device_status(NULL, NULL) == KD_ERR_INVALID_ARG, "status of a null workspace");

  if (failures == 0) printf("ok\n");
  return failures == 0 ? 0 : 1;
}
