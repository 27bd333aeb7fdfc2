/* Calls libfa through include/fa.h from plain C (no Python, no GPU needed):
 * every check below fails argument validation before the device is touched.
 * Prints one line per check; exits non-zero on the first mismatch. */
#include <stdio.h>
#include <string.h>

#include "fa.h"

static int expect(const char *what, int got, int want) {
  printf("%s: %d (%s)\n", what, got, fa_strerror(got));
  if (got != want) {
    printf("  expected %d\n", want);
    return 1;
  }
  return 0;
}

int main(void) {
  char *p = (char *)0x10000; /* a fake, 16-byte aligned device address */
  int bad = 0;
  bad |= expect("fwd NULL q", fa_fwd(NULL, p, p, p, (float *)p, 1, 1, 16, 64, 0.1f, 0, NULL),
                FA_ERR_NULL);
  bad |= expect("fwd d=96", fa_fwd(p, p, p, p, (float *)p, 1, 1, 16, 96, 0.1f, 0, NULL),
                FA_ERR_UNSUPPORTED_D);
  bad |= expect("fwd misaligned", fa_fwd(p + 2, p, p, p, (float *)p, 1, 1, 16, 64, 0.1f, 0, NULL),
                FA_ERR_ALIGN);
  bad |= expect("bwd N=0",
                fa_bwd(p, p, p, p, p, (float *)p, p, p, p, 1, 1, 0, 64, 0.1f, 1, p, 1 << 20, 0, NULL),
                FA_ERR_SHAPE);
  bad |= expect("decode Nq=9",
                fa_decode(p, p, p, p, (float *)p, NULL, 1, 1, 9, 64, 64, 64, 0.1f, 0, 0, NULL, 0, NULL),
                FA_ERR_SHAPE);
  bad |= expect("fp8 d=64",
                fa_fwd_fp8(p, p, p, (float *)p, (float *)p, (float *)p, p, (float *)p, 1, 1, 16, 64,
                           0.1f, 0, NULL),
                FA_ERR_UNSUPPORTED_D);
  bad |= expect("gemm K=0", fa_gemm(p, p, p, 4, 4, 0, 4, 4, 4, NULL, 0, NULL), FA_ERR_SHAPE);
  bad |= expect("selftest limit", fa_selftest_wait_timeout(0, NULL), FA_ERR_ARG);
  {
    int tn = 0, tm = 0, tiles_n = 0;
    bad |= expect("gemm tiles", fa_gemm_tiles(1792, 1792, 108, &tn, &tm, &tiles_n), FA_OK);
    if (tn != 128 || tm * tiles_n != 98) {
      printf("  tiles %d x %d of width %d, expected 98 of width 128\n", tm, tiles_n, tn);
      bad = 1;
    }
  }
  {
    int splits = 0, chunk = 0;
    bad |= expect("decode plan", fa_decode_plan(256, 1, 8192, 128, 0, 148, 2, &splits, &chunk), FA_OK);
    if (chunk % 64 != 0 || splits * chunk < 8192) {
      printf("  plan %d x %d does not cover 8192 keys\n", splits, chunk);
      bad = 1;
    }
  }
  {
    int items = 0, merged = 0, shift = 0;
    bad |= expect("fwd schedule", fa_fwd_schedule(2, 32, 4096, 1, 148, &items, &merged, &shift), FA_OK);
    if (items != 32 * 8 + 32 * 16 || merged != 32 || shift != 2) {
      printf("  %d items, %d merged heads, shift %d; expected 768, 32, 2\n", items, merged, shift);
      bad = 1;
    }
  }
  printf(bad ? "FAILED\n" : "OK\n");
  return bad;
}
