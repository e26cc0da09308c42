// Host run of the policy selection (block_sparse_long_exp_b200/csrc/
// msa_policy_unit.cuh) as the kernel uses it: per (query, group) the index
// query staged as float, every non-forced causal block scored, then the
// selection.  Reads a case written by tests/test_policy_select_cpu.py and
// writes sel [T, G, k].
#include <cstdint>
#include <cstdio>
#include <vector>

#include "msa_policy_unit.cuh"

template <class T>
static bool rd(FILE* f, std::vector<T>& v, size_t n) {
  v.resize(n);
  return fread(v.data(), sizeof(T), n, f) == n;
}

int main(int argc, char** argv) {
  if (argc != 3) return 2;
  FILE* f = fopen(argv[1], "rb");
  if (!f) return 2;
  int32_t hdr[9];
  if (fread(hdr, 4, 9, f) != 9) return 2;
  const int T = hdr[0], S = hdr[1], G = hdr[2], d_idx = hdr[3], k = hdr[4], B_k = hdr[5], batch = hdr[6],
            n_sink = hdr[7], n_local = hdr[8];
  std::vector<int32_t> cu_q, cu_k;
  std::vector<uint16_t> q_idx, k_idx;
  if (!rd(f, cu_q, batch + 1) || !rd(f, cu_k, batch + 1) || !rd(f, q_idx, (size_t)T * G * d_idx) ||
      !rd(f, k_idx, (size_t)S * d_idx))
    return 2;
  fclose(f);
  std::vector<int32_t> sel((size_t)T * G * k);
  std::vector<float> score(msa::kPolicyMaxBlocks);
  for (int b = 0; b < batch; ++b) {
    const int Tb = cu_q[b + 1] - cu_q[b], Sb = cu_k[b + 1] - cu_k[b];
    for (int i = 0; i < Tb; ++i) {
      const int64_t t = cu_q[b] + i, pos = (int64_t)Sb - Tb + i, lb = pos / B_k;
      for (int g = 0; g < G; ++g) {
        std::vector<float> qif(d_idx);
        for (int c = 0; c < d_idx; ++c) qif[c] = msa::pol_bf16(q_idx[(t * G + g) * d_idx + c]);
        const uint16_t* kirow = k_idx.data() + (int64_t)cu_k[b] * d_idx;
        if (lb + 1 > k)
          for (int64_t bb = 0; bb <= lb; ++bb)
            score[bb] = msa::pol_forced(bb, lb, n_sink, n_local) ? 0.f
                                                                 : msa::pol_block_score(qif.data(), kirow, d_idx, B_k,
                                                                                        bb, pos);
        msa::pol_select(score.data(), lb, k, n_sink, n_local, sel.data() + (t * G + g) * k);
      }
    }
  }
  FILE* o = fopen(argv[2], "wb");
  if (!o) return 2;
  fwrite(sel.data(), 4, sel.size(), o);
  fclose(o);
  return 0;
}
