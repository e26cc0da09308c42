// Prints the sliding-window baseline's blocks (block_sparse_long_exp_b200/
// csrc/msa_window.h, the rule the selection kernel runs) for every local
// block lb < 70, budget k in 1..9 and sink count 0..k-1: one line
// "lb k n_sink b0 b1 ... b(k-1)".
#include <cstdint>
#include <cstdio>

#include "msa_window.h"

int main() {
  int32_t out[16];
  for (int k = 1; k <= 9; ++k)
    for (int n_sink = 0; n_sink < k; ++n_sink)
      for (int64_t lb = 0; lb < 70; ++lb) {
        msa::window_blocks(lb, k, n_sink, out);
        printf("%lld %d %d", static_cast<long long>(lb), k, n_sink);
        for (int i = 0; i < k; ++i) printf(" %d", out[i]);
        printf("\n");
      }
  return 0;
}
