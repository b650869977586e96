/* A C program using libpa.so through include/pa.h only (no Python, no CUDA headers): the
 * host-side entry points that need no GPU.  Prints "ok" and exits 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "pa.h"

#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
      return 1;                                                  \
    }                                                            \
  } while (0)

int main(void) {
  CHECK(pa_version() == 101);
  CHECK(strlen(pa_strerror(PA_OK)) > 0);
  CHECK(strstr(pa_strerror(12345), "unknown") != NULL);

  /* workspace of the 8B-shaped batch: 256 sequences, 32 query heads, head_dim 128, 8192 tokens */
  size_t ws = pa_decode_workspace_size(256, 32, 128, 8192, 0);
  CHECK(ws >= (size_t)256 * 16 * 32 * 128 * 4); /* fp32 partial outputs of 16 partitions */
  CHECK(pa_decode_workspace_size(-1, 32, 128, 8192, 0) == 0);

  /* argument validation happens on the host, before any CUDA call: fake device addresses */
  void* fake = (void*)(uintptr_t)0x10000;
  const int32_t* ifake = (const int32_t*)fake;
  CHECK(pa_decode(fake, fake, fake, fake, ifake, ifake, 0, 32, 8, 128, 16, 0.088f, 512, 1000, PA_BF16, PA_BF16,
                  PA_BF16, 0, fake, 0, NULL) == PA_OK); /* no sequences: nothing to do */
  CHECK(pa_decode(fake, fake, fake, fake, ifake, ifake, 4, 6, 4, 128, 16, 0.088f, 512, 1000, PA_BF16, PA_BF16,
                  PA_BF16, 0, fake, 0, NULL) == PA_ERR_INVALID); /* heads not a multiple */
  CHECK(pa_decode(fake, fake, fake, fake, ifake, ifake, 4, 32, 8, 96, 16, 0.088f, 512, 1000, PA_BF16, PA_BF16,
                  PA_BF16, 0, fake, 0, NULL) == PA_ERR_UNSUPPORTED); /* head_dim 96 */
  CHECK(pa_decode(fake, fake, fake, fake, ifake, ifake, 4, 32, 8, 128, 16, 0.088f, 512, 1000, PA_BF16, PA_BF16,
                  PA_BF16, 0, fake, 100, NULL) == PA_ERR_WORKSPACE);
  CHECK(pa_decode_multi(fake, fake, fake, fake, ifake, ifake, 4, 0, 32, 8, 128, 16, 0.088f, 512, 1000, PA_BF16,
                        PA_BF16, PA_BF16, 0, fake, 0, NULL) == PA_ERR_INVALID); /* no query tokens */
  /* 5 members x 8 heads = 40 rows: the default option takes the tensor-core kernel (up to 64 rows),
     so the call passes the row check and stops at the missing workspace; the warp-MMA kernel
     holds 32 rows and refuses it */
  CHECK(pa_decode_prefix(fake, fake, fake, fake, ifake, ifake, 4, 64, 8, 128, 16, 0.088f, 512, 1000, PA_BF16,
                         PA_BF16, PA_BF16, 0, ifake, 1, 5, fake, 0, NULL) == PA_ERR_WORKSPACE);
  CHECK(pa_set_option(PA_OPT_WIDE_KERNEL, PA_WIDE_MMA) == PA_OK);
  CHECK(pa_decode_prefix(fake, fake, fake, fake, ifake, ifake, 4, 64, 8, 128, 16, 0.088f, 512, 1000, PA_BF16,
                         PA_BF16, PA_BF16, 0, ifake, 1, 5, fake, 0, NULL) == PA_ERR_UNSUPPORTED);
  CHECK(pa_copy_blocks(fake, fake, ifake, 1, 10, 4008, NULL, NULL) == PA_ERR_INVALID); /* not 16-byte units */
  CHECK(pa_selftest_wait_timeout(0, NULL) == PA_ERR_INVALID);
  /* the wide-item kernel option: its three values, nothing else */
  CHECK(pa_set_option(PA_OPT_WIDE_KERNEL, PA_WIDE_TCGEN05) == PA_OK);
  CHECK(pa_set_option(PA_OPT_WIDE_KERNEL, PA_WIDE_MMA) == PA_OK);
  CHECK(pa_set_option(PA_OPT_WIDE_KERNEL, PA_WIDE_AUTO) == PA_OK);
  CHECK(pa_set_option(PA_OPT_WIDE_KERNEL, 7) == PA_ERR_INVALID);
  CHECK(pa_set_option(99, PA_WIDE_MMA) == PA_ERR_INVALID);
  /* the item-split option: its two values, nothing else */
  CHECK(pa_set_option(PA_OPT_ITEM_SPLIT, PA_SPLIT_FIXED) == PA_OK);
  CHECK(pa_set_option(PA_OPT_ITEM_SPLIT, PA_SPLIT_ADAPTIVE) == PA_OK);
  CHECK(pa_set_option(PA_OPT_ITEM_SPLIT, 2) == PA_ERR_INVALID);
  puts("ok");
  return 0;
}
