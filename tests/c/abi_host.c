/*
 * The C ABI from a C11 program: the header compiles as C, the library links,
 * and the calls that need no GPU answer as declared (status strings, size
 * queries, argument errors returned on the host before any CUDA call).
 * Built and run by tests/test_abi.py.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "mala.h"

#define CHECK(c)                                                   \
  do {                                                             \
    if (!(c)) {                                                    \
      fprintf(stderr, "line %d: %s\n", __LINE__, #c);              \
      return 1;                                                    \
    }                                                              \
  } while (0)

int main(void) {
  /* any 16-byte-aligned address: argument checks never dereference it */
  void* p = (void*)(uintptr_t)256;
  float* f = (float*)p;

  CHECK(mala_version() >= 100);
  CHECK(strcmp(mala_status_string(MALA_OK), "MALA_OK") == 0);
  CHECK(strcmp(mala_status_string(MALA_ERR_TOO_LARGE), "MALA_ERR_TOO_LARGE") == 0);

  CHECK(mala_bwd_workspace_bytes(1, 2, 1000, 128) > 0);
  CHECK(mala_decode_workspace_bytes(2, 8, 2, 1000, 128) > 0);
  CHECK(mala_varlen_trace_words(4096, 131072) == (32 + 1024 + 31) / 32);

  CHECK(mala_fwd(p, p, p, p, f, NULL, 1, 1, 1, 256, 128, MALA_BF16, -1.0f, 128, 0.0f,
                 NULL, NULL, NULL) == MALA_ERR_INVALID_ARG);
  CHECK(mala_fwd(NULL, p, p, p, f, NULL, 1, 1, 1, 256, 128, MALA_BF16, 1.0f, 128, 0.0f,
                 NULL, NULL, NULL) == MALA_ERR_INVALID_ARG);
  CHECK(mala_fwd(p, p, p, p, f, NULL, 1, 1, 1, 256, 64, MALA_BF16, 1.0f, 128, 0.0f, NULL,
                 NULL, NULL) == MALA_ERR_UNSUPPORTED);
  CHECK(mala_fwd(p, p, p, p, f, NULL, 1, 4, 3, 256, 128, MALA_BF16, 1.0f, 128, 0.0f, NULL,
                 NULL, NULL) == MALA_ERR_INVALID_ARG);
  CHECK(mala_fwd(p, p, p, p, f, NULL, 1, 1, 1, 0, 128, MALA_BF16, 1.0f, 128, 0.0f, NULL,
                 NULL, NULL) == MALA_OK);

  CHECK(mala_bwd(p, p, p, p, NULL, p, f, p, p, p, p, 0, 1, 2, 2, 1000, 128, MALA_BF16,
                 1.0f, 128, 0.0f, NULL, NULL, NULL) == MALA_ERR_INVALID_ARG);

  CHECK(mala_decode(p, p, p, p, 2, 8, 3, 1000, 128, 1.0f, 0.0f, 0, p, 1 << 30, NULL, NULL,
                    NULL) == MALA_ERR_INVALID_ARG);
  CHECK(mala_decode(p, p, p, p, 2, 8, 2, 1000, 128, 1.0f, 0.0f, 2, p, 1 << 30, NULL, NULL,
                    NULL) == MALA_ERR_INVALID_ARG);
  CHECK(mala_decode_noalloc(p, p, p, p, 64, 64, 8, 32768, 128, 1.0f, 0.0f, NULL, NULL, NULL) ==
        MALA_ERR_TOO_LARGE);
  CHECK(MALA_DECODE_NOALLOC_SCRATCH_BYTES == (8u << 20));

  printf("ok\n");
  return 0;
}
