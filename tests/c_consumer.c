/* A plain C consumer of libint8mm.so: links against the library through
 * include/int8mm.h and calls the entry points that need no GPU (sizes, status
 * strings, argument validation that returns before any launch). Exit status 0
 * when every check holds; the failing check's line otherwise. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "int8mm.h"

#define CHECK(c)                                            \
  do {                                                      \
    if (!(c)) {                                             \
      fprintf(stderr, "check failed at line %d\n", __LINE__); \
      return __LINE__;                                      \
    }                                                       \
  } while (0)

int main(void) {
  /* fake, aligned device addresses: validation must refuse before touching them */
  void* A = (void*)(uintptr_t)(1u << 20);
  const size_t need = int8_mixed_matmul_workspace_size(64, 64, 64);
  CHECK(need > 0);
  CHECK(int8_mixed_matmul_workspace_size(4, 4, 20) == 0);
  CHECK(int8_mixed_matmul(A, A, A, A, 64, 64, 24, 6.0f, A, A, need, 0) == I8MM_ERR_ALIGNMENT);
  CHECK(int8_mixed_matmul(A, A, A, A, 64, 64, 64, -1.0f, A, A, need, 0) == I8MM_ERR_INVALID_ARG);
  CHECK(int8_mixed_matmul(A, A, A, A, 64, 64, 64, 6.0f, A, A, need - 1, 0) == I8MM_ERR_WORKSPACE);
  CHECK(int8_mixed_matmul(NULL, A, A, A, 0, 64, 64, 6.0f, NULL, NULL, 0, 0) == I8MM_OK);
  CHECK(int8_rotated_workspace_size(64, 64, 256) > 0);
  CHECK(int8_rotate_quantize_rows(A, 4, 256, 24, A, A, NULL, 0) == I8MM_ERR_INVALID_ARG);
  CHECK(strlen(int8_status_string(I8MM_ERR_TIMEOUT)) > 0);
  CHECK(strlen(int8_status_string(I8MM_OK)) > 0);
  printf("c consumer ok\n");
  return 0;
}
