// Host run of the index-alignment unit code (block_sparse_long_exp_b200/csrc/
// msa_kl_unit.cuh) exactly as the kernel uses it: per (query, group) the query
// heads, index query and log-sum-exps are staged as float, every thread of a
// CTA computes its partial sums, and the partials are merged.  Threads are run
// one after another, for a CTA of 128 threads and of 7 (another partition of
// the same support); then the gradient pass the same way, with the student's
// log-sum-exp from the forward.  Reads a case written by
// tests/test_kl_unit_cpu.py and writes, for both CTA sizes, kl[T, G], then
// dq_idx[T, G, d_idx], then dk_idx[S, d_idx].
#include <cstdint>
#include <cstdio>
#include <vector>

#include "msa_kl_unit.cuh"

template <class T>
static bool rd(FILE* f, std::vector<T>& v, size_t n) {
  v.resize(n);
  return fread(v.data(), sizeof(T), n, f) == n;
}

int main(int argc, char** argv) {
  if (argc != 3) return 2;
  FILE* f = fopen(argv[1], "rb");
  if (!f) return 2;
  int32_t hdr[10];
  float sc[2];
  if (fread(hdr, 4, 10, f) != 10 || fread(sc, 4, 2, f) != 2) return 2;
  const int T = hdr[0], S = hdr[1], H = hdr[2], G = hdr[3], d = hdr[4], d_idx = hdr[5], k = hdr[6], B_k = hdr[7],
            batch = hdr[8], dense = hdr[9];
  std::vector<int32_t> cu_q, cu_k, sel;
  std::vector<uint16_t> q, key, q_idx, k_idx;
  std::vector<float> lse;
  if (!rd(f, cu_q, batch + 1) || !rd(f, cu_k, batch + 1) || !rd(f, q, (size_t)T * H * d) ||
      !rd(f, key, (size_t)S * G * d) || !rd(f, q_idx, (size_t)T * G * d_idx) || !rd(f, k_idx, (size_t)S * d_idx) ||
      !rd(f, sel, (size_t)T * G * k) || !rd(f, lse, (size_t)T * H))
    return 2;
  fclose(f);
  const int Hg = H / G;
  std::vector<float> out((size_t)2 * T * G);
  std::vector<float> dq((size_t)2 * T * G * d_idx, 0.f), dk((size_t)2 * S * d_idx, 0.f);
  int bad_total = 0;
  for (int b = 0; b < batch; ++b) {
    const int Tb = cu_q[b + 1] - cu_q[b], Sb = cu_k[b + 1] - cu_k[b];
    for (int i = 0; i < Tb; ++i) {
      const int64_t t = cu_q[b] + i;
      for (int g = 0; g < G; ++g) {
        std::vector<float> qf(Hg * d), qif(d_idx), ls(Hg);
        for (int x = 0; x < Hg * d; ++x) qf[x] = msa::kl_bf16(q[(t * H + (int64_t)g * Hg) * d + x]);
        for (int x = 0; x < d_idx; ++x) qif[x] = msa::kl_bf16(q_idx[(t * G + g) * d_idx + x]);
        for (int x = 0; x < Hg; ++x) ls[x] = lse[t * H + (int64_t)g * Hg + x];
        msa::KlUnit u;
        u.qf = qf.data(); u.qif = qif.data(); u.lse = ls.data();
        u.krow = key.data() + (int64_t)cu_k[b] * G * d;
        u.kirow = k_idx.data() + (int64_t)cu_k[b] * d_idx;
        u.blocks = dense ? nullptr : sel.data() + (t * G + g) * k;
        u.nsel = k; u.Hg = Hg; u.d = d; u.d_idx = d_idx; u.G = G; u.g = g; u.B_k = B_k;
        u.pos = (int64_t)Sb - Tb + i;
        u.sm_scale = sc[0]; u.tau = sc[1]; u.dense = dense != 0;
        const int sizes[2] = {128, 7};
        for (int s = 0; s < 2; ++s) {
          std::vector<msa::KlPartial> parts(sizes[s]);
          int bad = 0;
          for (int tid = 0; tid < sizes[s]; ++tid) parts[tid] = msa::kl_thread(u, tid, sizes[s], &bad);
          bad_total += bad;
          float lse_z = 0.f;
          out[(size_t)s * T * G + t * G + g] = msa::kl_merge(parts.data(), sizes[s], &lse_z);
          float* dqu = dq.data() + ((size_t)s * T * G + t * G + g) * d_idx;
          float* dku = dk.data() + ((size_t)s * S + cu_k[b]) * d_idx;
          // each thread's own dq row, then the rows summed in thread order (as the kernel does)
          std::vector<float> rows((size_t)sizes[s] * d_idx, 0.f);
          for (int tid = 0; tid < sizes[s]; ++tid)
            msa::kl_grad_thread(u, lse_z, tid, sizes[s], rows.data() + (size_t)tid * d_idx, dku, &bad);
          for (int c = 0; c < d_idx; ++c) {
            float acc = 0.f;
            for (int tid = 0; tid < sizes[s]; ++tid) acc += rows[(size_t)tid * d_idx + c];
            dqu[c] = acc;
          }
          bad_total += bad;
        }
      }
    }
  }
  FILE* o = fopen(argv[2], "wb");
  if (!o) return 2;
  fwrite(out.data(), 4, out.size(), o);
  fwrite(dq.data(), 4, dq.size(), o);
  fwrite(dk.data(), 4, dk.size(), o);
  fclose(o);
  printf("bad %d\n", bad_total);
  return 0;
}
