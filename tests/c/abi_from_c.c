/* Calls the C ABI from plain C (no Python): the library's version and status
 * names, and argument validation that answers before any device work.
 * Exits 0 when every check holds; prints the first failing check otherwise. */
#include <stdio.h>
#include <string.h>

#include "fa_b200.h"

#define CHECK(cond)                                          \
  do {                                                       \
    if (!(cond)) {                                           \
      fprintf(stderr, "check failed: %s (line %d)\n", #cond, \
              __LINE__);                                     \
      return 1;                                              \
    }                                                        \
  } while (0)

int main(void) {
  /* 16-byte aligned addresses that validation never dereferences */
  const void *a = (const void *)0x10000;
  float *lse = (float *)0x10000;
  fa_mods none = FA_MODS_NONE;

  CHECK(strncmp(fa_version(), "fa_b200", 7) == 0);
  CHECK(strcmp(fa_status_string(FA_OK), "FA_OK") == 0);
  CHECK(strcmp(fa_status_string(FA_ERR_UNSUPPORTED), "FA_ERR_UNSUPPORTED") == 0);

  /* head dim 100 is not served */
  CHECK(fa_fwd(a, a, a, (void *)a, lse, 1, 16, 16, 4, 2, 100, FA_BF16, 0, 0.f, NULL,
               NULL, 0, NULL) == FA_ERR_UNSUPPORTED);
  CHECK(strlen(fa_last_error_message()) > 0);
  /* Hq not a multiple of Hkv */
  CHECK(fa_fwd(a, a, a, (void *)a, lse, 1, 16, 16, 4, 3, 128, FA_BF16, 0, 0.f, NULL,
               NULL, 0, NULL) == FA_ERR_INVALID);
  /* a negative soft-cap through the modifier entry point */
  none.softcap = -1.f;
  CHECK(fa_fwd_ex(a, a, a, (void *)a, lse, 1, 16, 16, 4, 2, 128, FA_BF16, 0, 0.f, NULL,
                  NULL, 0, &none, NULL) == FA_ERR_INVALID);
  /* varlen without cu_seqlens */
  CHECK(fa_fwd_varlen(a, a, a, (void *)a, lse, NULL, NULL, NULL, 2, 8, 8, 16, 16, 4, 2,
                      128, FA_BF16, 0, 0.f, NULL, 0, NULL) == FA_ERR_INVALID);
  /* split-KV host logic */
  CHECK(fa_splitkv_workspace_bytes(8, 1, 32, 128, 37) >= (size_t)37 * 8 * 32 * 129 * 4);
  CHECK(fa_splitkv_default_splits(8, 1, 131072, 32, 8, 128, 148) >= 16);
  /* merging partials: zero parts is invalid */
  CHECK(fa_combine_partials((const float *)a, (const float *)a, 0, 1, 1, 4, 128, FA_BF16,
                            (void *)a, lse, NULL) == FA_ERR_INVALID);
  printf("ok\n");
  return 0;
}
