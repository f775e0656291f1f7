/* Calls the host-only entry points of include/bsa.h from plain C11: builds a
 * log-linear pattern with the two-call protocol, validates it, copies it to
 * column-major, checks sizes and error codes.  Prints "ok" and exits 0 on
 * success; prints the failed check and exits 1 otherwise. */
#include <stdio.h>
#include <stdlib.h>

#include "bsa.h"

#define CHECK(cond)                                      \
  do {                                                   \
    if (!(cond)) {                                       \
      printf("failed: %s (line %d)\n", #cond, __LINE__); \
      return 1;                                          \
    }                                                    \
  } while (0)

int main(void) {
  const int32_t M = 8, H = 2;
  const int32_t anchors[3] = {0, 4, 7};
  bsa_pattern_desc d = {0};
  d.kind = BSA_LOGLINEAR;
  d.M = M;
  d.H = H;
  d.local_radius = 1;
  d.log_kmax = 2;
  d.n_anchors = 3;
  d.anchors = anchors;
  d.causal = 0;
  d.dilation = 1;

  int64_t nnz = -1;
  CHECK(bsa_build_pattern(&d, NULL, NULL, 0, &nnz) == BSA_OK);
  CHECK(nnz == 2 * 52); /* 52 stored blocks per head for M = 8, strides 1, 2, 4, anchors 0/4/7 */
  int32_t* row_ptr = (int32_t*)malloc(sizeof(int32_t) * (size_t)(H * M + 1));
  int32_t* col_idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)nnz);
  CHECK(bsa_build_pattern(&d, row_ptr, col_idx, nnz - 1, &nnz) == BSA_ERR_BUFFER_TOO_SMALL);
  CHECK(bsa_build_pattern(&d, row_ptr, col_idx, nnz, &nnz) == BSA_OK);
  CHECK(row_ptr[0] == 0 && row_ptr[H * M] == nnz);
  CHECK(bsa_validate_pattern(row_ptr, col_idx, nnz, H, M, 0) == BSA_OK);

  int32_t* col_ptr = (int32_t*)malloc(sizeof(int32_t) * (size_t)(H * M + 1));
  int32_t* row_idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)nnz);
  int64_t tnnz = -1;
  CHECK(bsa_transpose_pattern(row_ptr, col_idx, H, M, col_ptr, row_idx, nnz, &tnnz) == BSA_OK);
  CHECK(tnnz == nnz && col_ptr[H * M] == nnz);
  /* every (i, j) of the CSR appears as (j, i) in the copy */
  for (int32_t h = 0; h < H; ++h)
    for (int32_t i = 0; i < M; ++i)
      for (int32_t p = row_ptr[h * M + i]; p < row_ptr[h * M + i + 1]; ++p) {
        const int32_t j = col_idx[p];
        int found = 0;
        for (int32_t q = col_ptr[h * M + j]; q < col_ptr[h * M + j + 1]; ++q) found |= row_idx[q] == i;
        CHECK(found);
      }

  CHECK(bsa_topk_nnz(16, 128, 25, 0) == 16LL * 128 * 26);
  CHECK(bsa_topk_workspace_bytes(16, 4096, 64, 32) == 2u * 16 * 128 * 64 * 8);
  CHECK(bsa_backward_workspace_bytes(1, 2, 512) == 4u * 2 * 512 + 16u * 2 * 4);
  CHECK(bsa_forward(NULL, NULL, NULL, NULL, NULL, 1, 1, 256, 64, 32, 0.125f, 0, NULL, NULL, NULL) ==
        BSA_ERR_INVALID_ARG);
  CHECK(bsa_version() == 200);
  free(row_ptr);
  free(col_idx);
  free(col_ptr);
  free(row_idx);
  printf("ok\n");
  return 0;
}
