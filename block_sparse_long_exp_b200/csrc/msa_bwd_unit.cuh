// msa_bwd_unit.cuh — the Main Branch backward of one (query, group), in the two
// phases a CTA runs per chunk of its support: the per-token phase and the dq
// product.
//
// Softmax attention over the support J (the selected blocks' tokens cut at the
// query, or every causal token), differentiated as usual (MSA is trained end
// to end; the forward is yifor-blog "設計核心" item 2 / pnsm.cn sec. 2): for head
// h with saved lse_h, output o_h and upstream gradient dO_h,
//   P_j = exp(sm_scale q_h.k_j - lse_h),  dP_j = dO_h.v_j,  D_h = dO_h.o_h,
//   dS_j = P_j (dP_j - D_h),
//   dq_h = sm_scale sum_j dS_j k_j,  dk_j += sm_scale dS_j q_h,  dv_j += P_j dO_h.
// The support is numbered in ascending token order and cut into chunks of
// kBwdChunk tokens.  Phase 1 (one thread per token of the chunk) computes the
// token's dS for every head of the group, stages its key row, and adds its dk
// and dv rows (atomically on the device: other queries add to the same rows).
// Phase 2 (every thread, after a barrier) adds the chunk's share of
// dq = sm_scale dS . K to the thread's outputs.
//
// Plain fp32 arithmetic on bf16 bit patterns; compiled for the device by the
// kernel and for the host by a test, which replays a CTA phase by phase
// against an fp64 oracle.
#pragma once

#include <stdint.h>

#include <cmath>
#include <cstring>
#ifndef __CUDACC__
#define MSA_BWD_HD inline
#define MSA_BWD_HD_UNROLL
#else
#define MSA_BWD_HD __host__ __device__ __forceinline__
#define MSA_BWD_HD_UNROLL _Pragma("unroll")
#endif

namespace msa {

constexpr int kBwdChunk = 64;     // support tokens per chunk
constexpr int kBwdMaxHeads = 16;  // query heads per group (H / G) the unit code supports
constexpr int kBwdMaxBlocks = 64; // selected blocks (k <= 32) or dense blocks per pass of the block list

MSA_BWD_HD float bwd_bf16(uint16_t bits) {
  const uint32_t u = static_cast<uint32_t>(bits) << 16;
  float x;
#ifdef __CUDA_ARCH__
  x = __uint_as_float(u);
#else
  std::memcpy(&x, &u, 4);
#endif
  return x;
}

MSA_BWD_HD float bwd_exp(float x) {
#ifdef __CUDA_ARCH__
  return __expf(x);
#else
  return std::exp(x);
#endif
}

MSA_BWD_HD void bwd_add(float* dst, float v) {
#ifdef __CUDA_ARCH__
  atomicAdd(dst, v);
#else
  *dst += v;
#endif
}

// One (query, group): qf / dof the group's Hg query heads and upstream
// gradients as float [Hg * d]; lse / D per head [Hg]; krow / vrow the
// sequence's keys and values (bf16 bits, row j of group g at base + (j * G +
// g) * d); blocks the selected ids (ascending, -1 padding).
struct BwdUnit {
  const float* qf;
  const float* dof;
  const float* lse;
  const float* D;
  const uint16_t* krow;
  const uint16_t* vrow;
  const int32_t* blocks;
  int nsel, Hg, d, G, g, B_k;
  int64_t pos;
  float sm_scale;
  bool dense;
};

// The support as a list of token ranges: first[i] the first token of range i,
// base[i] the support tokens before it (base[n] = |J|).  Returns n (<= nsel or
// the causal block count; a dense support longer than kBwdMaxBlocks blocks is
// a single range).  A selected id past the query's block sets *bad and is
// left out.
MSA_BWD_HD int bwd_ranges(const BwdUnit& u, int64_t* first, int64_t* base, int* bad) {
  const int64_t lb = u.pos / u.B_k;
  int n = 0;
  base[0] = 0;
  if (u.dense) {
    first[0] = 0;
    base[1] = u.pos + 1;
    return 1;
  }
  for (int i = 0; i < u.nsel; ++i) {
    const int64_t b = u.blocks[i];
    if (b < 0) continue;
    if (b > lb) {
      *bad = 1;
      continue;
    }
    const int64_t j0 = b * u.B_k;
    const int64_t j1 = (b + 1) * u.B_k < u.pos + 1 ? (b + 1) * u.B_k : u.pos + 1;
    first[n] = j0;
    base[n + 1] = base[n] + (j1 - j0);
    ++n;
  }
  return n;
}

// Token of support position m (0 <= m < base[n]).
MSA_BWD_HD int64_t bwd_token(const int64_t* first, const int64_t* base, int n, int64_t m) {
  int i = 0;
  while (i + 1 < n && base[i + 1] <= m) ++i;
  return first[i] + (m - base[i]);
}

// Phase 1 for support token j: dS of every head into dS[h * kBwdChunk + slot],
// the key row (bf16 bits) into kstage[0 .. d), and the token's dk / dv rows
// (dk, dv: the gradients' rows of this sequence, float [S_b, G, d]).
MSA_BWD_HD void bwd_phase1(const BwdUnit& u, int64_t j, int slot, float* dS, uint16_t* kstage, float* dk, float* dv) {
  const uint16_t* kj = u.krow + (j * u.G + u.g) * u.d;
  const uint16_t* vj = u.vrow + (j * u.G + u.g) * u.d;
  float* dkj = dk + (j * u.G + u.g) * u.d;
  float* dvj = dv + (j * u.G + u.g) * u.d;
  // every head's score and dP, reading the key and value rows once
  float s[kBwdMaxHeads], dp[kBwdMaxHeads], p[kBwdMaxHeads], ds[kBwdMaxHeads];
MSA_BWD_HD_UNROLL
  for (int h = 0; h < kBwdMaxHeads; ++h) s[h] = dp[h] = p[h] = ds[h] = 0.f;
  for (int c = 0; c < u.d; ++c) {
    kstage[c] = kj[c];
    const float kc = bwd_bf16(kj[c]), vc = bwd_bf16(vj[c]);
MSA_BWD_HD_UNROLL
    for (int h = 0; h < kBwdMaxHeads; ++h)
      if (h < u.Hg) {
        s[h] += u.qf[h * u.d + c] * kc;
        dp[h] += u.dof[h * u.d + c] * vc;
      }
  }
MSA_BWD_HD_UNROLL
  for (int h = 0; h < kBwdMaxHeads; ++h)
    if (h < u.Hg) {
      p[h] = bwd_exp(u.sm_scale * s[h] - u.lse[h]);
      ds[h] = p[h] * (dp[h] - u.D[h]);
      dS[h * kBwdChunk + slot] = ds[h];
    }
  // the token's dk / dv rows: one atomic add per element, summed over the heads first
  for (int c = 0; c < u.d; ++c) {
    float gk = 0.f, gv = 0.f;
MSA_BWD_HD_UNROLL
    for (int h = 0; h < kBwdMaxHeads; ++h)
      if (h < u.Hg) {
        gk += ds[h] * u.qf[h * u.d + c];
        gv += p[h] * u.dof[h * u.d + c];
      }
    bwd_add(dkj + c, u.sm_scale * gk);
    bwd_add(dvj + c, gv);
  }
}

// Phase 2: output o = h * d + c of dq gets sum over the chunk's cnt tokens of
// dS[h][slot] * k[slot][c] (the caller scales by sm_scale at the end).
MSA_BWD_HD float bwd_phase2(const BwdUnit& u, const float* dS, const uint16_t* kst, int cnt, int o) {
  const int h = o / u.d, c = o - h * u.d;
  float acc = 0.f;
  for (int s = 0; s < cnt; ++s) acc += dS[h * kBwdChunk + s] * bwd_bf16(kst[s * u.d + c]);
  return acc;
}

}  // namespace msa

#undef MSA_BWD_HD
#undef MSA_BWD_HD_UNROLL
