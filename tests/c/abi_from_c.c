/* A plain C99 caller of libfattn: compiles against include/fattn.h alone (no CUDA or
 * PyTorch headers), links the shared library and exercises the calls that need no GPU —
 * workspace sizes, status strings, and host-side validation, which returns before any
 * CUDA call.  Exit status 0 when every check holds; the first failing check is printed. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fattn.h"

static int failures = 0;

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

int main(void) {
  /* a 16-byte aligned address that is never dereferenced: validation fails first */
  void* p = (void*)(uintptr_t)4096;
  float* f = (float*)p;
  const int* cu = (const int*)p;

  CHECK(strcmp(fa_status_string(FA_OK), "ok") == 0);
  CHECK(strcmp(fa_status_string(FA_ERR_TIMEOUT), "device wait timed out") == 0);
  CHECK(fa_last_error() != NULL);

  /* D (fp32 per row and head) and the fp32 dQ sums ([rows, H, d]), each in 256-byte units */
  CHECK(fa_bwd_workspace_size(2, 16384, 32, 128) ==
        (size_t)2 * 16384 * 32 * 4 + (size_t)2 * 16384 * 32 * 128 * 4);
  CHECK(fa_bwd_workspace_size(1, 3, 1, 64) == 256 + (size_t)3 * 64 * 4);
  CHECK(fa_varlen_bwd_workspace_size(896, 32, 128) ==
        (size_t)896 * 32 * 4 + (size_t)896 * 32 * 128 * 4);

  /* head_dim 96 is not built; an unknown dtype; null and misaligned pointers */
  CHECK(fa_fwd(p, p, p, p, f, 1, 128, 1, 96, 0.1f, 0, FA_BF16, NULL) == FA_ERR_UNSUPPORTED);
  CHECK(fa_fwd(p, p, p, p, f, 1, 128, 1, 64, 0.1f, 0, 7, NULL) == FA_ERR_UNSUPPORTED);
  CHECK(fa_fwd(NULL, p, p, p, f, 1, 128, 1, 64, 0.1f, 1, FA_FP16, NULL) == FA_ERR_INVALID_ARG);
  CHECK(fa_fwd((char*)p + 2, p, p, p, f, 1, 128, 1, 64, 0.1f, 1, FA_BF16, NULL) ==
        FA_ERR_INVALID_ARG);
  CHECK(fa_fwd(p, p, p, p, f, -1, 128, 1, 64, 0.1f, 1, FA_BF16, NULL) == FA_ERR_INVALID_ARG);
  CHECK(fa_varlen_fwd(p, p, p, p, f, cu, NULL, 128, 128, 1, 64, 0.1f, 1, 1, 128, 128, FA_BF16,
                      NULL) == FA_ERR_INVALID_ARG);
  CHECK(fa_bwd(p, p, p, p, p, f, p, p, p, 1, 128, 1, 64, 0.1f, 1, p, 16, FA_BF16, NULL) ==
        FA_ERR_INVALID_ARG); /* workspace smaller than fa_bwd_workspace_size */

  if (failures == 0) printf("abi_from_c: all checks passed\n");
  return failures == 0 ? 0 : 1;
}
