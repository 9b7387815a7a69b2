/* Plain-C user of the cpattn ABI: compiles against include/cpattn.h with a C compiler
 * (no CUDA or C++ headers) and checks calls that must fail argument validation before any
 * CUDA work, so it runs on a machine without a GPU.  Exit status 0 = all checks passed. */
#include <stdint.h>
#include <stdio.h>

#include "cpattn.h"

static int failures = 0;

static void expect(const char* what, int got, int want) {
  if (got != want) {
    fprintf(stderr, "%s: got %d (%s), want %d (%s)\n", what, got, cpattn_status_str(got), want,
            cpattn_status_str(want));
    ++failures;
  }
}

int main(void) {
  /* 16-byte aligned addresses that are never dereferenced: every call below is refused
   * by the host-side checks */
  void* a = (void*)(uintptr_t)0x100000;
  void* b = (void*)(uintptr_t)0x2000000;
  float* l = (float*)(uintptr_t)0x3000000;
  expect("fwd: Sq = 0", cpattn_fwd(a, a, a, b, l, 1, 2, 0, 8, 128, 0.1f, CPATTN_BF16,
                                   CPATTN_BF16, NULL),
         CPATTN_ERR_SHAPE);
  expect("fwd: null q", cpattn_fwd(NULL, a, a, b, l, 1, 2, 8, 8, 128, 0.1f, CPATTN_BF16,
                                   CPATTN_BF16, NULL),
         CPATTN_ERR_NULL);
  expect("merge: D = 0", cpattn_merge(a, l, a, l, b, l, 1, 2, 8, 0, CPATTN_BF16, NULL),
         CPATTN_ERR_SHAPE);
  expect("seq2head: H % P", cpattn_seq2head(a, b, 3, 4, 16, 128, 2, NULL), CPATTN_ERR_SHAPE);
  expect("head2seq: elem_bytes", cpattn_head2seq(a, b, 2, 4, 16, 128, 3, NULL), CPATTN_ERR_SHAPE);
  expect("rmsnorm: D = 96", cpattn_rmsnorm(a, b, l, 10, 96, 1e-6f, 1.0f, NULL), CPATTN_ERR_SHAPE);
  expect("rmsnorm: no rows", cpattn_rmsnorm(NULL, NULL, NULL, 0, 128, 1e-6f, 1.0f, NULL),
         CPATTN_OK);
  /* pure host arithmetic: the split-KV workspace size and the wave model's split choice */
  if (cpattn_fwd_split_workspace(1, 16, 512, 128, 4, CPATTN_BF16) == 0) {
    fprintf(stderr, "split workspace: zero bytes\n");
    ++failures;
  }
  if (cpattn_split_suggest(1, 16, 512, 44160) < 4) {
    fprintf(stderr, "split suggestion for a 512-row query slice below 4\n");
    ++failures;
  }
  if (failures == 0) printf("cpattn C ABI: all checks passed (version 0x%x)\n", cpattn_version());
  return failures == 0 ? 0 : 1;
}
