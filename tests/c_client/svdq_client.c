/* A plain C client of the library: compiled against include/svdq.h as C99 and linked to
 * libsvdq.so, it calls the entry points through their C signatures.  Without a GPU it exercises
 * what needs none: the version and size queries, argument errors reported before any launch, and
 * empty batches (M = 0), which launch nothing.  Exit status 0 when every check holds. */
#include <stdio.h>
#include <string.h>

#include "svdq.h"

static int failures = 0;

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

int main(void) {
  CHECK(svdq_version() > 0);
  CHECK(strcmp(svdq_status_string(SVDQ_OK), "SVDQ_OK") == 0);
  CHECK(strcmp(svdq_status_string(SVDQ_ERR_CHECK), "SVDQ_ERR_CHECK") == 0);

  /* sizes: ceil(rows / 128) * 128 * K / 16 (NVFP4), * K / 32 (MXFP4) */
  CHECK(svdq_sf_bytes(1, 64) == 128 * 4);
  CHECK(svdq_sf_bytes(129, 128) == 256 * 8);
  CHECK(svdq_sf_bytes(16, 100) == 0);
  CHECK(svdq_mx_sf_bytes(1, 128) == 128 * 4);
  CHECK(svdq_quantize_act_workspace_bytes(4608, 3072, 0) == 0);
  CHECK(svdq_quantize_act_workspace_bytes(4608, 3072, 32) > 0);
  CHECK(svdq_linear_gelu_quantize_workspace_bytes(4608, 12288, 32) == (size_t)48 * 4608 * 32 * 4);

  /* empty batches: valid, nothing launched, NULL buffers allowed */
  CHECK(svdq_quantize_act(NULL, 0, 256, NULL, 1.0f, NULL, 32, 1.0f, NULL, NULL, NULL, NULL, 0, NULL) == SVDQ_OK);
  CHECK(svdq_linear(NULL, NULL, 1.0f, NULL, NULL, 1.0f, NULL, NULL, 32, NULL, NULL, 0, 0, 512, 256, NULL) == SVDQ_OK);
  CHECK(svdq_linear_mx(NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL, NULL, 0, 0, 256, 256, NULL) == SVDQ_OK);

  /* argument errors, reported before anything touches a device */
  CHECK(svdq_quantize_act(NULL, -1, 256, NULL, 1.0f, NULL, 0, 1.0f, NULL, NULL, NULL, NULL, 0, NULL) ==
        SVDQ_ERR_INVALID_ARG);
  CHECK(svdq_quantize_act(NULL, 0, 100, NULL, 1.0f, NULL, 0, 1.0f, NULL, NULL, NULL, NULL, 0, NULL) ==
        SVDQ_ERR_UNSUPPORTED_SHAPE);
  CHECK(svdq_linear(NULL, NULL, 1.0f, NULL, NULL, 1.0f, NULL, NULL, 8, NULL, NULL, 0, 16, 64, 64, NULL) ==
        SVDQ_ERR_UNSUPPORTED_SHAPE);
  CHECK(svdq_linear(NULL, NULL, 1.0f, NULL, NULL, 1.0f, NULL, NULL, 0, NULL, NULL, 0, 16, 64, 64, NULL) ==
        SVDQ_ERR_INVALID_ARG);
  CHECK(svdq_linear_mx(NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL, NULL, 0, 16, 64, 192, NULL) ==
        SVDQ_ERR_UNSUPPORTED_SHAPE);
  CHECK(svdq_gelu_bf16(NULL, 0, NULL, NULL) == SVDQ_OK);
  CHECK(svdq_gelu_bf16(NULL, -1, NULL, NULL) == SVDQ_ERR_INVALID_ARG);

  uint64_t hits = 1, misses = 1;
  svdq_map_cache_stats(&hits, &misses);
  CHECK(hits == 0 && misses == 0);
  CHECK(svdq_build_flags() == 0 || svdq_build_flags() == 1);

  if (failures) {
    fprintf(stderr, "%d check(s) failed\n", failures);
    return 1;
  }
  printf("c client ok\n");
  return 0;
}
