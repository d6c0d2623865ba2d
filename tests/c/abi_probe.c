/*
 * abi_probe.c - the C ABI of libfa_b200.so called from plain C99, with no
 * CUDA header: include/fa_b200.h must compile as C, and every entry point must
 * link and answer.  Only calls that fail an argument check are made, so
 * nothing is ever launched and the probe runs the same with or without a GPU.
 * Prints "OK" and exits 0 when every check holds.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fa_b200.h"

static int fails = 0;

#define CHECK(expr, want)                                                         \
  do {                                                                            \
    long long got_ = (long long)(expr);                                           \
    if (got_ != (long long)(want)) {                                              \
      printf("FAIL %s = %lld, expected %lld\n", #expr, got_, (long long)(want)); \
      fails++;                                                                    \
    }                                                                             \
  } while (0)

int main(void) {
  /* 16-byte aligned addresses that are never dereferenced: every call below
     returns before any launch */
  void* A = (void*)(uintptr_t)0x10000;
  void* MIS = (void*)(uintptr_t)0x10008;
  float* L = (float*)A;
  const size_t rows = (size_t)2 * 3 * 1000;
  const size_t ws = fa_bwd_workspace_size(2, 3, 1000, 64);
  int s;

  CHECK(ws, ((rows * 64 * 4 + 255) / 256) * 256 + ((rows * 4 + 255) / 256) * 256);
  CHECK(fa_bwd_workspace_size(1, 1, 1, 96), 0);
  CHECK(fa_bwd_workspace_size(1, 32768, 1024, 64), 0); /* 2^31 elements */
  CHECK(FA_BWD_NOALLOC_SCRATCH_BYTES, (size_t)32 << 20);

  CHECK(fa_fwd(NULL, A, A, A, L, 1, 1, 128, 64, 1, 0.125f, 1, NULL), FA_ERR_NULL);
  CHECK(fa_fwd(A, A, A, A, L, 1, 1, 128, 96, 1, 0.125f, 1, NULL), FA_ERR_HEADDIM);
  CHECK(fa_fwd(A, A, A, A, L, 1, 32768, 1024, 64, 1, 0.125f, 1, NULL), FA_ERR_SHAPE);
  CHECK(fa_fwd(A, A, A, A, L, 1, 1, 128, 64, 2, 0.125f, 1, NULL), FA_ERR_ARG);
  CHECK(fa_fwd(A, A, A, MIS, L, 1, 1, 128, 64, 1, 0.125f, 1, NULL), FA_ERR_ALIGN);
  CHECK(fa_fwd(A, A, A, A, L, 1, 1, 128, 64, 1, 0.125f, 7, NULL), FA_ERR_FIXMODE);
  CHECK(fa_fwd_debug(A, A, A, A, L, NULL, NULL, NULL, 1, 1, 1, 128, 64, 1, 0.125f, 1, FA_ELEM_BF16, NULL),
        FA_ERR_NULL);
  CHECK(fa_fwd_debug(A, A, A, A, L, NULL, (int32_t*)A, NULL, 1, 4, 3, 128, 64, 1, 0.125f, 1, FA_ELEM_F16, NULL),
        FA_ERR_SHAPE);
  CHECK(fa_fwd_ex(A, A, A, A, L, 1, 1, 1, 128, 64, 1, 0.125f, 6, FA_ELEM_F16, NULL), FA_ERR_FIXMODE);
  CHECK(fa_fwd_ex(A, A, A, A, L, 1, 4, 3, 128, 64, 1, 0.125f, 1, FA_ELEM_BF16, NULL), FA_ERR_SHAPE);
  CHECK(fa_fwd_ex(A, A, A, A, L, 1, 4, 2, 128, 64, 1, 0.125f, 1, 9, NULL), FA_ERR_ARG);
  CHECK(fa_fwd_ex(A, A, A, A, L, 1, 4, 2, 128, 64, 1, 0.125f, 1, FA_ELEM_F16 + 1, NULL), FA_ERR_ARG);

  CHECK(fa_bwd(A, A, A, A, L, A, A, A, A, A, ws - 1, 2, 3, 1000, 64, 1, 0.125f, NULL), FA_ERR_WORKSPACE);
  CHECK(fa_bwd(A, A, A, A, L, A, A, A, A, NULL, ws, 2, 3, 1000, 64, 1, 0.125f, NULL), FA_ERR_WORKSPACE);
  CHECK(fa_bwd_ex(A, A, A, A, L, A, MIS, A, A, A, ws, 2, 3, 3, 1000, 64, 1, 0.125f, FA_ELEM_F16, NULL),
        FA_ERR_ALIGN);
  CHECK(fa_bwd_ex(A, A, A, A, L, A, A, A, A, A, ws, 2, 3, 2, 1000, 64, 1, 0.125f, FA_ELEM_BF16, NULL),
        FA_ERR_SHAPE);
  CHECK(fa_bwd_ex(A, A, A, A, L, A, A, A, A, A, ws, 2, 3, 3, 1000, 64, 1, 0.125f, -1, NULL), FA_ERR_ARG);
  CHECK(fa_bwd_preprocess(A, NULL, A, ws, 2, 3, 1000, 64, NULL), FA_ERR_NULL);
  CHECK(fa_bwd_main(A, A, A, L, A, A, A, A, ws, 2, 3, 1000, 64, 1, -1.0f, NULL), FA_ERR_ARG);
  CHECK(fa_bwd_finish(A, A, ws, 2, 3, 1000, 32, 0.125f, NULL), FA_ERR_HEADDIM);
  CHECK(fa_bwd_noalloc(A, A, A, A, L, A, A, A, A, 1, 1, 129056, 64, 1, 0.125f, NULL), FA_ERR_SCRATCH_LIMIT);
  CHECK(fa_watchdog_selftest(0, NULL), FA_ERR_ARG);

  for (s = FA_ERR_BUILD; s <= FA_OK; ++s) {
    const char* msg = fa_status_string(s);
    if (!msg || !strlen(msg) || !strcmp(msg, "unknown status")) {
      printf("FAIL status string for %d\n", s);
      fails++;
    }
  }
  if (strcmp(fa_status_string(12345), "unknown status") != 0) {
    printf("FAIL status string for an unknown code\n");
    fails++;
  }
  printf("%s\n", fails ? "FAILED" : "OK");
  return fails != 0;
}
