// msa_kl_unit.cuh — the index-alignment target of one (query, group), split
// over threads: the per-thread partial sums and their merge.
//
// The Index Branch is trained by a KL divergence that pulls its distribution
// towards the Main Branch's attention on the selected support, with the
// gradient kept away from the backbone (pnsm.cn "MiniMax Sparse Attention：
// 一篇读懂百万上下文时代的稀疏注意力工程化路线", sec. 4 and sec. 5; yhxrc.cn
// sec. 二).  Over the support J of query t and group g:
//   teacher  P_j = mean over the group's heads h of exp(sm_scale q_h.k_j - lse_h)
//            (lse_h: the main branch's log-sum-exp over J, so each head's
//            distribution sums to 1 and so does their mean),
//   student  Q_j = softmax_J(z), z_j = tau q_idx.k_idx_j,
//   KL(P || Q) = sum_j P_j log P_j - sum_j P_j z_j + log sum_j exp(z_j).
// The three sums split over any partition of J: each thread keeps A = sum
// P log P, B = sum P z and a (max, sum) pair for the log-sum-exp; the merge
// adds A and B and combines the pairs.  J is the selected blocks' tokens cut
// at the query (sparse form) or every token 0..pos (the dense form used while
// the index branch warms up on full attention).
//
// Plain fp32 arithmetic on bf16 bit patterns; compiled for the device by the
// kernel and for the host by a test, which checks it against an fp64 oracle.
#pragma once

#include <stdint.h>

#include <cmath>
#include <cstring>
#ifndef __CUDACC__
#define MSA_KL_HD inline
#define MSA_KL_HD_UNROLL
#else
#define MSA_KL_HD __host__ __device__ __forceinline__
#define MSA_KL_HD_UNROLL _Pragma("unroll")
#endif

namespace msa {

constexpr int kKlMaxHeads = 16;   // query heads per group (H / G) the unit code supports

struct KlPartial {
  float A;   // sum of P log P
  float B;   // sum of P z
  float m;   // running max of z
  float l;   // sum of exp(z - m)
};

MSA_KL_HD float kl_bf16(uint16_t bits) {
  const uint32_t u = static_cast<uint32_t>(bits) << 16;
  float x;
#ifdef __CUDA_ARCH__
  x = __uint_as_float(u);
#else
  std::memcpy(&x, &u, 4);
#endif
  return x;
}

MSA_KL_HD float kl_exp(float x) {
#ifdef __CUDA_ARCH__
  return __expf(x);
#else
  return std::exp(x);
#endif
}

MSA_KL_HD float kl_log(float x) {
#ifdef __CUDA_ARCH__
  return __logf(x);
#else
  return std::log(x);
#endif
}

// Eight consecutive bf16 values (16 bytes, 16-byte aligned) as floats.
MSA_KL_HD void kl_load8(const uint16_t* p, float* out) {
  uint16_t v[8];
#ifdef __CUDA_ARCH__
  *reinterpret_cast<uint4*>(v) = *reinterpret_cast<const uint4*>(p);
#else
  std::memcpy(v, p, 16);
#endif
MSA_KL_HD_UNROLL
  for (int i = 0; i < 8; ++i) out[i] = kl_bf16(v[i]);
}

// Everything one (query, group) needs.  qf: the group's Hg query heads as
// float [Hg * d]; qif: its index query as float [d_idx]; lse: the heads'
// log-sum-exps over J [Hg]; krow / kirow: the sequence's keys (bf16 bits,
// key row j of group g at krow + (j * G + g) * d) and index keys (kirow +
// j * d_idx); blocks: the selected block ids (ascending, -1 padding).
struct KlUnit {
  const float* qf;
  const float* qif;
  const float* lse;
  const uint16_t* krow;
  const uint16_t* kirow;
  const int32_t* blocks;
  int nsel, Hg, d, d_idx, G, g, B_k;
  int64_t pos;
  float sm_scale, tau;
  bool dense;
};

// Visits this thread's support tokens n = tid, tid + nthreads, ... (tokens
// numbered in ascending order) with f(j, P_j, raw index score, index-key
// row).  A block id outside 0..pos / B_k sets *bad and is skipped, so no read
// leaves the sequence.
template <class F>
MSA_KL_HD void kl_for_tokens(const KlUnit& u, int tid, int nthreads, int* bad, F&& f) {
  const int64_t lb = u.pos / u.B_k;
  const int nblk = u.dense ? static_cast<int>(lb) + 1 : u.nsel;
  int64_t base = 0;   // support tokens before this block
  for (int i = 0; i < nblk; ++i) {
    const int64_t b = u.dense ? i : u.blocks[i];
    if (b < 0) continue;
    if (b > lb) {
      *bad = 1;
      continue;
    }
    const int64_t j0 = b * u.B_k;
    const int64_t j1 = (b + 1) * u.B_k < u.pos + 1 ? (b + 1) * u.B_k : u.pos + 1;
    const int64_t n0 = base;
    base += j1 - j0;
    // first token of this block that belongs to thread tid
    int64_t first = (tid - n0) % nthreads;
    if (first < 0) first += nthreads;
    for (int64_t j = j0 + first; j < j1; j += nthreads) {
      const uint16_t* kj = u.krow + (j * u.G + u.g) * u.d;
      // every head's score, reading the key row once (kKlMaxHeads sums in registers)
      // (rows are read 16 bytes at a time; each head's sum still runs over c in order)
      float s[kKlMaxHeads];
MSA_KL_HD_UNROLL
      for (int h = 0; h < kKlMaxHeads; ++h) s[h] = 0.f;
      for (int c0 = 0; c0 < u.d; c0 += 8) {
        float kc[8];
        kl_load8(kj + c0, kc);
MSA_KL_HD_UNROLL
        for (int e = 0; e < 8; ++e)
MSA_KL_HD_UNROLL
          for (int h = 0; h < kKlMaxHeads; ++h)
            if (h < u.Hg) s[h] += u.qf[h * u.d + c0 + e] * kc[e];
      }
      float pbar = 0.f;
MSA_KL_HD_UNROLL
      for (int h = 0; h < kKlMaxHeads; ++h)
        if (h < u.Hg) pbar += kl_exp(u.sm_scale * s[h] - u.lse[h]);
      pbar *= 1.f / u.Hg;
      const uint16_t* kij = u.kirow + j * u.d_idx;
      float zs = 0.f;
      for (int c0 = 0; c0 < u.d_idx; c0 += 8) {
        float ki[8];
        kl_load8(kij + c0, ki);
MSA_KL_HD_UNROLL
        for (int e = 0; e < 8; ++e) zs += u.qif[c0 + e] * ki[e];
      }
      f(j, pbar, zs, kij);
    }
  }
}

// This thread's partial sums of the KL.
MSA_KL_HD KlPartial kl_thread(const KlUnit& u, int tid, int nthreads, int* bad) {
  KlPartial r{0.f, 0.f, -INFINITY, 0.f};
  kl_for_tokens(u, tid, nthreads, bad, [&](int64_t, float pbar, float zs, const uint16_t*) {
    const float z = u.tau * zs;
    if (pbar > 0.f) r.A += pbar * kl_log(pbar);
    r.B += pbar * z;
    if (z > r.m) {
      r.l = r.l * kl_exp(r.m - z) + 1.f;
      r.m = z;
    } else {
      r.l += kl_exp(z - r.m);
    }
  });
  return r;
}

// KL = sum A - sum B + log-sum-exp merged over the partials; *lse_z (if
// given) receives the student's log-sum-exp log sum_j exp(z_j).
MSA_KL_HD float kl_merge(const KlPartial* p, int n, float* lse_z = nullptr) {
  float A = 0.f, B = 0.f, m = -INFINITY;
  for (int i = 0; i < n; ++i) {
    A += p[i].A;
    B += p[i].B;
    if (p[i].l > 0.f && p[i].m > m) m = p[i].m;
  }
  float l = 0.f;
  for (int i = 0; i < n; ++i)
    if (p[i].l > 0.f) l += p[i].l * kl_exp(p[i].m - m);
  if (lse_z != nullptr) *lse_z = l > 0.f ? m + kl_log(l) : -INFINITY;
  return l > 0.f ? A - B + m + kl_log(l) : 0.f;
}

// Four consecutive floats added to dst (16-byte aligned): one vector reduction
// on the device (other queries add to the same key rows), plain adds on the host.
MSA_KL_HD void kl_add4(float* dst, float a, float b, float c, float d) {
#ifdef __CUDA_ARCH__
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
#else
  dst[0] += a; dst[1] += b; dst[2] += c; dst[3] += d;
#endif
}

// Gradient of KL(P || Q) with the teacher P held constant, over this thread's
// support tokens: with w_j = tau (Q_j - P_j), Q_j = exp(z_j - lse_z),
//   dq[c]              += w_j k_idx[j][c]   (the index query's gradient)
//   dk[j * d_idx + c]  += w_j q_idx[c]      (the index keys' gradient)
// dq is this thread's own accumulator row (the caller sums the rows of all
// threads); dk rows are added with kl_add4 (dk points at the sequence's first
// key row of the fp32 [S, d_idx] gradient).
MSA_KL_HD void kl_grad_thread(const KlUnit& u, float lse_z, int tid, int nthreads, float* dq, float* dk, int* bad) {
  kl_for_tokens(u, tid, nthreads, bad, [&](int64_t j, float pbar, float zs, const uint16_t* kij) {
    const float w = u.tau * (kl_exp(u.tau * zs - lse_z) - pbar);
    for (int c0 = 0; c0 < u.d_idx; c0 += 8) {
      float ki[8];
      kl_load8(kij + c0, ki);
MSA_KL_HD_UNROLL
      for (int e = 0; e < 8; ++e) dq[c0 + e] += w * ki[e];
      float* dkr = dk + j * u.d_idx + c0;
      kl_add4(dkr, w * u.qif[c0], w * u.qif[c0 + 1], w * u.qif[c0 + 2], w * u.qif[c0 + 3]);
      kl_add4(dkr + 4, w * u.qif[c0 + 4], w * u.qif[c0 + 5], w * u.qif[c0 + 6], w * u.qif[c0 + 7]);
    }
  });
}

}  // namespace msa

#undef MSA_KL_HD
#undef MSA_KL_HD_UNROLL
