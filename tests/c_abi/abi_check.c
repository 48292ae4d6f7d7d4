/* A plain C caller of libpbs.so, compiled against include/pbs.h by
 * tests/test_abi_host.py: if a declaration in the header drifts from what
 * this file passes, it stops compiling.  Every call below is rejected on the
 * host (before any CUDA call), so it runs without a GPU.  Exit status 0 and
 * the line "abi ok" mean every entry point returned the documented code. */
#include <stdio.h>
#include <string.h>

#include "pbs.h"

static int failures = 0;

static void expect(const char* what, int got, int want) {
  if (got != want) {
    printf("FAIL %s: got %d want %d (%s)\n", what, got, want, pbs_get_last_error());
    ++failures;
  }
}

int main(void) {
  pbs_tensor q, k, v, o;
  memset(&q, 0, sizeof q);
  q.ptr = (void*)0x1000; q.B = 1; q.H = 4; q.N = 1024; q.D = 128; q.sN = 128; q.sH = 1024 * 128; q.sB = 4 * 1024 * 128;
  k = q; k.H = 1; k.sB = 1024 * 128;
  v = k;
  o = q;
  int32_t* dummy = (int32_t*)0x2000;
  const char* ver = pbs_version();
  if (!ver || strncmp(ver, "pbs", 3) != 0) { printf("FAIL version\n"); ++failures; }

  expect("permute null Q", pbs_permute(NULL, &k, 128, 512, 0, dummy, NULL, 0, NULL), PBS_ERR_INVALID_ARG);
  expect("permute null perm", pbs_permute(&q, &k, 128, 512, 0, NULL, NULL, 0, NULL), PBS_ERR_INVALID_ARG);
  expect("permute blk", pbs_permute(&q, &k, 96, 512, 0, dummy, NULL, 0, NULL), PBS_ERR_UNSUPPORTED);
  expect("permute_noalloc null K", pbs_permute_noalloc(&q, NULL, 128, 512, 0, dummy, NULL), PBS_ERR_INVALID_ARG);
  expect("permute_segmented n_sink", pbs_permute_segmented(&q, &k, 128, 512, -1, dummy, NULL, 0, NULL),
         PBS_ERR_INVALID_ARG);
  expect("select mode", pbs_select(&q, &k, dummy, 128, 512, 7, 0.1, 0, 0, dummy, dummy, 8, NULL, 0, NULL),
         PBS_ERR_INVALID_ARG);
  expect("select capacity", pbs_select(&q, &k, dummy, 128, 512, PBS_SELECT_TOPK, 0.5, 0, 0, dummy, dummy, 1, NULL, 0,
                                       NULL), PBS_ERR_CAPACITY);
  if (pbs_select_capacity(1024, 128, 512, PBS_SELECT_TAU, 0.9, 0, 0) != 4) { printf("FAIL capacity\n"); ++failures; }
  if (pbs_workspace_size(PBS_OP_PERMUTE, NULL, &k, 128, 512) != 0) { printf("FAIL ws null\n"); ++failures; }
  if (pbs_workspace_size(PBS_OP_PERMUTE, &q, &k, 128, 512) != 512) { printf("FAIL ws permute\n"); ++failures; }
  expect("attn null V", pbs_attn_fwd(&q, &k, NULL, dummy, dummy, dummy, 4, 128, 512, NULL, 0.088f, &o, NULL, NULL,
                                     NULL, 0, NULL), PBS_ERR_INVALID_ARG);
  expect("attn scale", pbs_attn_fwd(&q, &k, &v, dummy, dummy, dummy, 4, 128, 512, NULL, -1.0f, &o, NULL, NULL, NULL, 0,
                                    NULL), PBS_ERR_INVALID_ARG);
  expect("attn_early_stop tau", pbs_attn_fwd_early_stop(&q, &k, &v, dummy, dummy, dummy, 4, 128, 512, -1.0f, 0.088f,
                                                        &o, NULL, NULL, NULL), PBS_ERR_INVALID_ARG);
  expect("attn_ex flags", pbs_attn_fwd_ex(&q, &k, &v, dummy, dummy, dummy, 4, 128, 512, 0x100u, NULL, 0.0f, 0.088f,
                                          &o, NULL, NULL, NULL), PBS_ERR_INVALID_ARG);
  pbs_test_inject_timeout(0u);
  if (failures == 0) printf("abi ok\n");
  return failures == 0 ? 0 : 1;
}
