/* Plain-C client of include/fa.h: compiled with a C99 compiler and linked
 * against libfa_b200.so by tests/test_c_client.py.  It exercises only the
 * calls that need no GPU (argument validation happens before any CUDA call),
 * so it runs on a machine without one.  Exit status 0 = every check passed. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fa.h"

static int failures = 0;

static void expect(int got, int want, const char* what) {
  if (got != want) {
    fprintf(stderr, "%s: got %d (%s), want %d\n", what, got, fa_status_string(got), want);
    ++failures;
  }
}

int main(void) {
  /* a 16-byte aligned address that is never dereferenced */
  void* a16 = (void*)(uintptr_t)(1u << 20);
  float* l16 = (float*)a16;

  expect(fa_abi_version() >> 16, 1, "ABI major version");
  if (strncmp(fa_status_string(FA_ERR_TIMEOUT), "FA_ERR_TIMEOUT", 14) != 0) ++failures;
  if (strcmp(fa_status_string(12345), "FA_ERR_UNKNOWN") != 0) ++failures;

  expect(fa_fwd(a16, a16, a16, a16, l16, -1, 2, 10, 10, 64, -1.0f, 0, FA_LAYOUT_BHND, FA_DTYPE_BF16, NULL),
         FA_ERR_INVALID_ARG, "negative B");
  expect(fa_fwd(a16, a16, a16, a16, l16, 1, 2, 10, 10, 96, -1.0f, 0, FA_LAYOUT_BHND, FA_DTYPE_BF16, NULL),
         FA_ERR_UNSUPPORTED, "head dim 96");
  expect(fa_fwd(a16, a16, a16, a16, l16, 1, 2, 10, 10, 64, -1.0f, 0, 7, FA_DTYPE_BF16, NULL),
         FA_ERR_INVALID_ARG, "bad layout");
  expect(fa_fwd((char*)a16 + 8, a16, a16, a16, l16, 1, 2, 10, 10, 64, -1.0f, 0, FA_LAYOUT_BSND, FA_DTYPE_FP16,
                NULL),
         FA_ERR_MISALIGNED, "misaligned q");
  expect(fa_fwd(NULL, NULL, NULL, NULL, NULL, 1, 2, 0, 10, 64, -1.0f, 1, FA_LAYOUT_BHND, FA_DTYPE_BF16, NULL),
         FA_OK, "empty problem is a no-op");
  expect(fa_fwd_gqa(a16, a16, a16, a16, l16, 1, 6, 4, 10, 10, 128, -1.0f, 0, FA_LAYOUT_BHND, FA_DTYPE_BF16, NULL),
         FA_ERR_INVALID_ARG, "Hkv not dividing H");
  expect(fa_fwd_noalloc(a16, a16, a16, a16, l16, 1, 2, 10, 0, 64, -1.0f, 0, FA_LAYOUT_BHND, FA_DTYPE_BF16, NULL),
         FA_ERR_INVALID_ARG, "empty key set");

  expect(fa_fwd_paged(a16, a16, a16, (const int*)a16, a16, l16, 1, 4, 2, 10, 100, 64, 24, 8, 4, -1.0f, 0,
                      FA_LAYOUT_BSND, FA_DTYPE_BF16, NULL),
         FA_ERR_INVALID_ARG, "paged block size not a power of two");
  expect(fa_fwd_paged(a16, a16, a16, (const int*)a16, a16, l16, 1, 4, 2, 10, 100, 64, 32, 8, 4, -1.0f, 0,
                      FA_LAYOUT_BSND, FA_DTYPE_FP32, NULL),
         FA_ERR_UNSUPPORTED, "paged fp32");

  {
    int splits = 0;
    int64_t ws = -1;
    expect(fa_splitkv_plan(1, 40, 1, 8192, 128, 5, 148, &splits, &ws), FA_OK, "split-KV plan");
    expect(splits, 5, "split-KV plan: slices");
    if (ws != (int64_t)5 * 40 * 129 * 4) ++failures;
  }
  expect(fa_fwd_splitkv(a16, a16, a16, a16, l16, 1, 4, 2, 1, 1000, 128, -1.0f, 0, a16, 1 << 20, FA_LAYOUT_BSND,
                        FA_DTYPE_FP32, NULL),
         FA_ERR_UNSUPPORTED, "split-KV fp32");
  expect(fa_fwd_paged_splitkv(a16, a16, a16, (const int*)a16, a16, l16, 1, 4, 2, 1, 1000, 128, 128, 9, 7, -1.0f, 0,
                              a16, 1 << 20, FA_LAYOUT_BSND, FA_DTYPE_BF16, NULL),
         FA_ERR_INVALID_ARG, "paged split-KV short table");

  uint32_t prev = fa_set_wait_timeout_us(5000);
  expect((int)fa_set_wait_timeout_us(prev), 5000, "timeout setting round trip");

  if (failures == 0) printf("c client ok\n");
  return failures == 0 ? 0 : 1;
}
