/* Plain-C use of the boundary (no PyTorch, no CUDA headers): host-side calls
 * that need no GPU -- the version string, workspace sizing and argument
 * checks.  Built and run by tests/test_abi_cpu.py; exits 0 when every check
 * holds. */
#include <stdio.h>
#include <string.h>

#include "msa.h"

static int fails = 0;
#define CHECK(cond)                                         \
  do {                                                      \
    if (!(cond)) {                                          \
      fprintf(stderr, "check failed: %s\n", #cond);         \
      ++fails;                                              \
    }                                                       \
  } while (0)

int main(void) {
  const char* v = msa_version();
  CHECK(v != NULL && strstr(v, "sm_100a") != NULL);

  msa_shape_t shape = {64, 4, 128, 64, 128, 16, 0.08838834764831845f};
  /* packed description of one 4096-token sequence; the offsets are only
     read by kernels, so host pointers are enough for sizing */
  int32_t cu[2] = {0, 4096};
  msa_varlen_t seqs = {1, 4096, 4096, 0, 4096, 4096, cu, cu};
  CHECK(msa_index_topk_workspace_size(&shape, &seqs) >= 256);
  CHECK(msa_sparse_attn_workspace_size(&shape, &seqs, 0) > 0);
  CHECK(msa_sparse_attn_workspace_size(&shape, &seqs, 1024) < msa_sparse_attn_workspace_size(&shape, &seqs, 0));
  CHECK(msa_dense_attn_workspace_size(&shape, &seqs) >= 256);

  msa_shape_t bad = shape;
  bad.d = 96;
  CHECK(msa_index_topk_workspace_size(&bad, &seqs) == 0);
  CHECK(msa_index_topk(&shape, &seqs, NULL, NULL, NULL, NULL, 0, NULL) == MSA_ERR_INVALID_ARG);
  CHECK(msa_index_topk(&bad, &seqs, cu, cu, cu, cu, 1 << 20, NULL) == MSA_ERR_UNSUPPORTED);

  int32_t prev = msa_set_tile_threshold(0);
  CHECK(msa_set_tile_threshold(prev) == 0);

  if (fails == 0) printf("abi_host ok: %s\n", v);
  return fails == 0 ? 0 : 1;
}
