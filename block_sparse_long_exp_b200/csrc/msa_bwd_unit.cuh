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
// kBwdChunk tokens whose key and value rows are staged first.  Per chunk:
// bwd_pds gives P and dS of one (token, head) from the staged rows;
// bwd_kv_cols gives one column of a token's dk and dv rows, summed over the
// heads (added atomically on the device: other queries add to the same rows);
// bwd_phase2 adds the chunk's share of dq = sm_scale dS . K to one output.
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

// Staged key / value rows: bf16 pairs as 32-bit words, row r at r * rw words
// (rw = d / 2 + 1: the pad word puts consecutive rows in different banks).
MSA_BWD_HD float bwd_lo(uint32_t w) { return bwd_bf16(static_cast<uint16_t>(w & 0xffffu)); }
MSA_BWD_HD float bwd_hi(uint32_t w) { return bwd_bf16(static_cast<uint16_t>(w >> 16)); }

// P and dS of tokens t0 .. t0 + nt - 1 (chunk slots; nt <= 2) and heads
// h0 .. h0 + nh - 1 (nh <= kBwdPdsHeads) from the staged rows, written to P /
// dS at [h * stride + slot].  Each (token, head) sum runs over c in ascending
// order, so the tiling does not change the result.
constexpr int kBwdPdsHeads = 4;
constexpr int kBwdPdsTokens = 2;
MSA_BWD_HD void bwd_pds(const BwdUnit& u, const uint32_t* kst, const uint32_t* vst, int rw, int t0, int nt, int h0,
                        int nh, float* P, float* dS, int stride) {
  float s[kBwdPdsTokens][kBwdPdsHeads], dp[kBwdPdsTokens][kBwdPdsHeads];
MSA_BWD_HD_UNROLL
  for (int a = 0; a < kBwdPdsTokens; ++a)
MSA_BWD_HD_UNROLL
    for (int i = 0; i < kBwdPdsHeads; ++i) s[a][i] = dp[a][i] = 0.f;
  const int t1 = nt > 1 ? t0 + 1 : t0;
  for (int w = 0; w < u.d / 2; ++w) {
    const uint32_t k0 = kst[t0 * rw + w], k1 = kst[t1 * rw + w];
    const uint32_t v0 = vst[t0 * rw + w], v1 = vst[t1 * rw + w];
    const float kc[2][2] = {{bwd_lo(k0), bwd_hi(k0)}, {bwd_lo(k1), bwd_hi(k1)}};
    const float vc[2][2] = {{bwd_lo(v0), bwd_hi(v0)}, {bwd_lo(v1), bwd_hi(v1)}};
MSA_BWD_HD_UNROLL
    for (int i = 0; i < kBwdPdsHeads; ++i) {
      if (i >= nh) continue;
      const float* qh = u.qf + (h0 + i) * u.d + 2 * w;
      const float* oh = u.dof + (h0 + i) * u.d + 2 * w;
      const float q0 = qh[0], q1 = qh[1], o0 = oh[0], o1 = oh[1];
MSA_BWD_HD_UNROLL
      for (int a = 0; a < kBwdPdsTokens; ++a) {
        s[a][i] += q0 * kc[a][0];
        s[a][i] += q1 * kc[a][1];
        dp[a][i] += o0 * vc[a][0];
        dp[a][i] += o1 * vc[a][1];
      }
    }
  }
MSA_BWD_HD_UNROLL
  for (int a = 0; a < kBwdPdsTokens; ++a)
MSA_BWD_HD_UNROLL
    for (int i = 0; i < kBwdPdsHeads; ++i)
      if (a < nt && i < nh) {
        const int h = h0 + i, slot = t0 + a;
        const float p = bwd_exp(u.sm_scale * s[a][i] - u.lse[h]);
        P[h * stride + slot] = p;
        dS[h * stride + slot] = p * (dp[a][i] - u.D[h]);
      }
}

// Column c of one token's dk and dv rows, summed over the heads: P and dS hold
// the token's values at [h * stride + slot].
MSA_BWD_HD void bwd_kv_cols(const BwdUnit& u, const float* P, const float* dS, int stride, int slot, int c, float* gk,
                            float* gv) {
  float k_ = 0.f, v_ = 0.f;
MSA_BWD_HD_UNROLL
  for (int h = 0; h < kBwdMaxHeads; ++h)
    if (h < u.Hg) {
      k_ += dS[h * stride + slot] * u.qf[h * u.d + c];
      v_ += P[h * stride + slot] * u.dof[h * u.d + c];
    }
  *gk = u.sm_scale * k_;
  *gv = v_;
}

// dq outputs (h, c0 .. c0 + 7) of one chunk: acc[e] += sum over the chunk's cnt
// tokens, in order, of dS[h][slot] * k[slot][c0 + e] (the caller scales by
// sm_scale at the end).
MSA_BWD_HD void bwd_phase2(const BwdUnit& u, const float* dS, const uint32_t* kst, int rw, int cnt, int h, int c0,
                           float* acc) {
  for (int s = 0; s < cnt; ++s) {
    const float ds = dS[h * kBwdChunk + s];
    const uint32_t* kr = kst + s * rw + c0 / 2;
MSA_BWD_HD_UNROLL
    for (int j = 0; j < 4; ++j) {
      const uint32_t w = kr[j];
      acc[2 * j] += ds * bwd_lo(w);
      acc[2 * j + 1] += ds * bwd_hi(w);
    }
  }
}

}  // namespace msa

#undef MSA_BWD_HD
#undef MSA_BWD_HD_UNROLL
