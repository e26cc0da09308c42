// msa_policy_unit.cuh — the scored selection policies the MSA pages compare the
// final rule with, for one (query, group): forced sink blocks and a forced
// local window, the rest of the k blocks by block score (pnsm.cn "MiniMax
// Sparse Attention：一篇读懂百万上下文时代的稀疏注意力工程化路线", sec. 3 and the
// forced sink / local ablation of its table; yhxrc.cn sec. 二: early versions
// forced the first block and a local window, the final rule only the current
// block).
//
//   forced = {0 .. n_sink-1} ∪ {lb-n_local+1 .. lb}, cut to 0 .. lb
//   sel    = every causal block when lb + 1 <= k, else forced ∪ the best
//            k - |forced| other causal blocks by (score desc, id asc)
// with a block's score the largest raw index score <q_idx, k_idx_j> over its
// tokens (NaN ranks as -inf).  n_sink = 0, n_local = 1 is the final rule.
//
// Plain fp32 arithmetic on bf16 bit patterns; compiled for the device by the
// kernel and for the host by a test, which checks it against the fp64 oracle.
#pragma once

#include <stdint.h>

#include <cmath>
#include <cstring>
#ifndef __CUDACC__
#define MSA_POL_HD inline
#else
#define MSA_POL_HD __host__ __device__ __forceinline__
#endif

namespace msa {

constexpr int kPolicyMaxBlocks = 8192;   // causal blocks per query (1M tokens at B_k = 128)
constexpr int kPolicyMaxK = 32;

MSA_POL_HD float pol_bf16(uint16_t bits) {
  const uint32_t u = static_cast<uint32_t>(bits) << 16;
  float x;
#ifdef __CUDA_ARCH__
  x = __uint_as_float(u);
#else
  std::memcpy(&x, &u, 4);
#endif
  return x;
}

MSA_POL_HD bool pol_forced(int64_t b, int64_t lb, int n_sink, int n_local) {
  return b < n_sink || b > lb - n_local;
}

// Score of block b for the index query qif [d_idx] over the index keys kirow
// (bf16 bits, row j at kirow + j * d_idx): the largest dot product over the
// block's tokens up to pos; NaN counts as -inf.
MSA_POL_HD float pol_block_score(const float* qif, const uint16_t* kirow, int d_idx, int B_k, int64_t b,
                                 int64_t pos) {
  float m = -INFINITY;
  const int64_t j1 = (b + 1) * B_k < pos + 1 ? (b + 1) * B_k : pos + 1;
  for (int64_t j = b * B_k; j < j1; ++j) {
    const uint16_t* kj = kirow + j * d_idx;
    float s = 0.f;
    // the row is read 16 bytes at a time (d_idx is a multiple of 8); the sum runs over c in order
    for (int c0 = 0; c0 < d_idx; c0 += 8) {
      uint16_t v[8];
#ifdef __CUDA_ARCH__
      *reinterpret_cast<uint4*>(v) = *reinterpret_cast<const uint4*>(kj + c0);
#else
      std::memcpy(v, kj + c0, 16);
#endif
      for (int e = 0; e < 8; ++e) s += qif[c0 + e] * pol_bf16(v[e]);
    }
    if (s > m) m = s;   // a NaN score never wins
  }
  return m;
}

// The forced blocks of a query in block lb, ascending (at most k of them).
MSA_POL_HD int pol_forced_list(int64_t lb, int n_sink, int n_local, int32_t* f) {
  int n = 0;
  for (int64_t b = 0; b <= lb; ++b) {
    if (b >= n_sink) {
      const int64_t w0 = lb - n_local + 1 > b ? lb - n_local + 1 : b;   // jump to the local window
      for (int64_t c = w0; c <= lb; ++c) f[n++] = static_cast<int32_t>(c);
      return n;
    }
    f[n++] = static_cast<int32_t>(b);
  }
  return n;
}

// The selection from the block scores score[0 .. lb] into out[0 .. k) (ascending
// ids, -1 padded).
MSA_POL_HD void pol_select(const float* score, int64_t lb, int k, int n_sink, int n_local, int32_t* out) {
  int n = 0;
  if (lb + 1 <= k) {
    for (int64_t b = 0; b <= lb; ++b) out[n++] = static_cast<int32_t>(b);
    for (; n < k; ++n) out[n] = -1;
    return;
  }
  int32_t f[kPolicyMaxK];
  const int nf = pol_forced_list(lb, n_sink, n_local, f);
  const int m = k - nf;   // blocks chosen by score
  // best m candidates by (score desc, id asc): insertion into a short sorted list
  int32_t top[kPolicyMaxK];
  float top_s[kPolicyMaxK];
  int nt = 0;
  for (int64_t b = 0; b <= lb && m > 0; ++b) {
    if (pol_forced(b, lb, n_sink, n_local)) continue;
    const float s = score[b] == score[b] ? score[b] : -INFINITY;
    // ids arrive ascending, so an equal score stays behind the ones kept
    int pos = nt;
    while (pos > 0 && top_s[pos - 1] < s) --pos;
    if (pos >= m) continue;
    const int last = nt < m ? nt : m - 1;
    for (int i = last; i > pos; --i) {
      top[i] = top[i - 1];
      top_s[i] = top_s[i - 1];
    }
    top[pos] = static_cast<int32_t>(b);
    top_s[pos] = s;
    if (nt < m) ++nt;
  }
  // forced and chosen blocks, sorted by id (at most k of them)
  for (int i = 0; i < nf; ++i) out[n++] = f[i];
  for (int i = 0; i < nt; ++i) {
    int p = n++;
    while (p > 0 && out[p - 1] > top[i]) {
      out[p] = out[p - 1];
      --p;
    }
    out[p] = top[i];
  }
  for (; n < k; ++n) out[n] = -1;
}

}  // namespace msa

#undef MSA_POL_HD
