/* Plain C99 client of include/fa.h: compiled and linked against libfa.so by
 * tests/test_c_header.py.  It only makes calls that return before touching a
 * GPU (size queries, status strings, argument errors), so it runs without one.
 * Prints one line per check; exit status 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fa.h"

static int failures = 0;

static void expect(int cond, const char* what) {
  printf("%s %s\n", cond ? "ok" : "FAIL", what);
  if (!cond) ++failures;
}

int main(void) {
  /* a 16-byte aligned address that is never dereferenced */
  void* a = (void*)(uintptr_t)(1u << 20);
  float* lse = (float*)a;

  expect(strncmp(fa_status_string(FA_OK), "FA_OK", 5) == 0, "status string of FA_OK");
  expect(strncmp(fa_status_string(FA_ERR_TIMEOUT), "FA_ERR_TIMEOUT", 14) == 0, "status string of FA_ERR_TIMEOUT");

  expect(fa_bwd_workspace_size(1, 32, 4096, 128) > 0, "backward workspace size");
  expect(fa_bwd_workspace_size(1, 1, 16, 96) == 0, "backward workspace size, unsupported D");
  expect(fa_decode_workspace_size(8, 32, 2, 128) > 0, "decode workspace size");
  expect(fa_decode_num_splits(8, 8, 8192) >= 1, "decode split count");

  expect(fa_fwd(a, a, a, a, lse, 1, 1, 16, 96, 0.125f, 0, FA_BF16, NULL) == FA_ERR_UNSUPPORTED, "fa_fwd, D = 96");
  expect(fa_fwd(a, a, a, a, lse, 1, 1, 16, 64, 0.0f, 0, FA_BF16, NULL) == FA_ERR_INVALID_ARG, "fa_fwd, scale 0");
  expect(fa_fwd(a, a, a, a, lse, 0, 1, 16, 64, 0.125f, 1, FA_FP16, NULL) == FA_OK, "fa_fwd, empty batch");
  expect(fa_fwd_dropout(a, a, a, a, lse, 1, 1, 16, 64, 0.125f, 0, FA_BF16, 1.0f, 1, 0, NULL) == FA_ERR_INVALID_ARG,
         "fa_fwd_dropout, p = 1");
  expect(fa_decode(a, a, a, (const int*)a, a, lse, 2, 8, 3, 100, 64, 0.125f, FA_BF16, 2, a, 1 << 20, NULL) ==
             FA_ERR_INVALID_ARG,
         "fa_decode, Hq not a multiple of Hkv");
  expect(fa_bwd(a, a, a, a, a, lse, a, a, a, 1, 1, 64, 64, 0.125f, 1, FA_BF16, 0, a, 16, NULL) == FA_ERR_INVALID_ARG,
         "fa_bwd, workspace too small");
  return failures == 0 ? 0 : 1;
}
