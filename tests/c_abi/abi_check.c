/* A C program against include/ssm_scan.h and libssmscan.so: the ABI as a C
 * caller sees it.  It needs no GPU: every call below must return its
 * documented status before any launch.  Exit status 0 when all hold. */
#include <stdint.h>
#include <stdio.h>

#include "ssm_scan.h"

static int failures = 0;

static void expect(const char *what, ssm_status got, ssm_status want) {
  if (got != want) {
    fprintf(stderr, "%s: got %d (%s), want %d (%s)\n", what, (int)got, ssm_status_string(got),
            (int)want, ssm_status_string(want));
    ++failures;
  }
}

int main(void) {
  ssm_shape s = {2, 16, 64, 16, SSM_BF16, SSM_PATH_AUTO, 0, 0};
  void *p = (void *)(uintptr_t)256; /* never dereferenced: every call fails its checks first */
  float *f = (float *)(uintptr_t)256;

  if (ssm_scan_version() < 100) ++failures;
  expect("null shape", ssm_scan_fwd(NULL, p, p, f, p, p, NULL, NULL, NULL, 1, NULL, p, NULL, p, 1 << 20, NULL),
         SSM_ERR_INVALID_ARG);
  ssm_shape bad = s;
  bad.dstate = 65;
  expect("dstate 65", ssm_scan_fwd(&bad, p, p, f, p, p, NULL, NULL, NULL, 1, NULL, p, NULL, p, 1 << 20, NULL),
         SSM_ERR_UNSUPPORTED);
  expect("null y", ssm_scan_fwd(&s, p, p, f, p, p, NULL, NULL, NULL, 1, NULL, NULL, NULL, p, 1 << 20, NULL),
         SSM_ERR_INVALID_ARG);
  ssm_shape one = s;
  one.seqlen = 2;
  expect("step with seqlen 2", ssm_scan_step(&one, p, p, f, p, p, NULL, NULL, NULL, 1, f, p, NULL),
         SSM_ERR_INVALID_ARG);
  expect("conv width 9", ssm_causal_conv1d(2, 16, 64, 9, SSM_BF16, p, f, NULL, NULL, 1, p, NULL, NULL),
         SSM_ERR_UNSUPPORTED);
  ssm_shape tokf = s;
  tokf.flags = SSM_FLAG_TOKEN_MAJOR;
  tokf.io_dtype = SSM_F32;
  expect("fp32 token-major backward", ssm_scan_bwd(&tokf, p, p, f, p, p, NULL, NULL, NULL, 1, NULL, p, NULL, p, p,
                                                   f, p, p, NULL, NULL, NULL, NULL, p, 1 << 20, NULL),
         SSM_ERR_UNSUPPORTED);
  ssm_shape empty = s;
  empty.batch = 0;
  expect("empty forward", ssm_scan_fwd(&empty, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, NULL, NULL,
                                       NULL, NULL, 0, NULL),
         SSM_OK);
  if (ssm_scan_fwd_workspace_bytes(&bad) != 0) ++failures;
  if (failures) return 1;
  printf("C ABI checks passed\n");
  return 0;
}
