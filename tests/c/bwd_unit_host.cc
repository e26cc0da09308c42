// Host replay of the Main Branch backward CTA (block_sparse_long_exp_b200/
// csrc/msa_bwd_unit.cuh) exactly as msa_attn_bwd.cu runs it: per (query,
// group) the staged query heads, upstream gradients, log-sum-exps and D =
// dO.o; the support's token ranges; then per chunk of kBwdChunk tokens phase 1
// for every token of the chunk and phase 2 for every dq output.  Reads a case
// written by tests/test_bwd_unit_cpu.py; writes dq [T, H, d], dk and dv
// [S, G, d] as float.
#include <cstdint>
#include <cstdio>
#include <vector>

#include "msa_bwd_unit.cuh"

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
  float sm;
  if (fread(hdr, 4, 9, f) != 9 || fread(&sm, 4, 1, f) != 1) return 2;
  const int T = hdr[0], S = hdr[1], H = hdr[2], G = hdr[3], d = hdr[4], k = hdr[5], B_k = hdr[6], batch = hdr[7],
            dense = hdr[8];
  std::vector<int32_t> cu_q, cu_k, sel;
  std::vector<uint16_t> q, key, val, out, dout;
  std::vector<float> lse;
  if (!rd(f, cu_q, batch + 1) || !rd(f, cu_k, batch + 1) || !rd(f, q, (size_t)T * H * d) ||
      !rd(f, key, (size_t)S * G * d) || !rd(f, val, (size_t)S * G * d) || !rd(f, sel, (size_t)T * G * k) ||
      !rd(f, out, (size_t)T * H * d) || !rd(f, lse, (size_t)T * H) || !rd(f, dout, (size_t)T * H * d))
    return 2;
  fclose(f);
  const int Hg = H / G;
  std::vector<float> dq((size_t)T * H * d, 0.f), dk((size_t)S * G * d, 0.f), dv((size_t)S * G * d, 0.f);
  int bad_total = 0;
  for (int b = 0; b < batch; ++b) {
    const int Tb = cu_q[b + 1] - cu_q[b], Sb = cu_k[b + 1] - cu_k[b];
    for (int i = 0; i < Tb; ++i) {
      const int64_t t = cu_q[b] + i;
      for (int g = 0; g < G; ++g) {
        const int64_t row0 = (t * H + (int64_t)g * Hg) * d;
        std::vector<float> qf(Hg * d), dof(Hg * d), ls(Hg), Ds(Hg, 0.f), dS(Hg * msa::kBwdChunk),
            P(Hg * msa::kBwdChunk);
        const int rw = d / 2 + 1;
        std::vector<uint32_t> kst(msa::kBwdChunk * rw), vst(msa::kBwdChunk * rw);
        for (int x = 0; x < Hg * d; ++x) {
          qf[x] = msa::bwd_bf16(q[row0 + x]);
          dof[x] = msa::bwd_bf16(dout[row0 + x]);
        }
        for (int h = 0; h < Hg; ++h) {
          ls[h] = lse[t * H + (int64_t)g * Hg + h];
          for (int c = 0; c < d; ++c) Ds[h] += dof[h * d + c] * msa::bwd_bf16(out[row0 + (int64_t)h * d + c]);
        }
        msa::BwdUnit u;
        u.qf = qf.data(); u.dof = dof.data(); u.lse = ls.data(); u.D = Ds.data();
        u.krow = key.data() + (int64_t)cu_k[b] * G * d;
        u.vrow = val.data() + (int64_t)cu_k[b] * G * d;
        u.blocks = dense ? nullptr : sel.data() + (t * G + g) * k;
        u.nsel = k; u.Hg = Hg; u.d = d; u.G = G; u.g = g; u.B_k = B_k;
        u.pos = (int64_t)Sb - Tb + i;
        u.sm_scale = sm; u.dense = dense != 0;
        int64_t first[msa::kBwdMaxBlocks], base[msa::kBwdMaxBlocks + 1];
        int bad = 0;
        const int n = msa::bwd_ranges(u, first, base, &bad);
        bad_total += bad;
        float* dk_seq = dk.data() + (int64_t)cu_k[b] * G * d;
        float* dv_seq = dv.data() + (int64_t)cu_k[b] * G * d;
        std::vector<float> acc(Hg * d, 0.f);
        for (int64_t c0 = 0; c0 < base[n]; c0 += msa::kBwdChunk) {
          const int cnt = base[n] - c0 < msa::kBwdChunk ? static_cast<int>(base[n] - c0) : msa::kBwdChunk;
          int64_t tok[msa::kBwdChunk];
          // stage the chunk's key and value rows (bf16 pairs as words, padded rows)
          for (int s = 0; s < cnt; ++s) {
            tok[s] = msa::bwd_token(first, base, n, c0 + s);
            const uint16_t* kr = u.krow + (tok[s] * G + g) * d;
            const uint16_t* vr = u.vrow + (tok[s] * G + g) * d;
            for (int w = 0; w < d / 2; ++w) {
              kst[s * rw + w] = (uint32_t)kr[2 * w] | ((uint32_t)kr[2 * w + 1] << 16);
              vst[s * rw + w] = (uint32_t)vr[2 * w] | ((uint32_t)vr[2 * w + 1] << 16);
            }
          }
          // the kernel's tiling: token pairs x head groups
          for (int t0 = 0; t0 < cnt; t0 += msa::kBwdPdsTokens)
            for (int h0 = 0; h0 < Hg; h0 += msa::kBwdPdsHeads)
              msa::bwd_pds(u, kst.data(), vst.data(), rw, t0, cnt - t0 < 2 ? cnt - t0 : 2, h0,
                           Hg - h0 < msa::kBwdPdsHeads ? Hg - h0 : msa::kBwdPdsHeads, P.data(), dS.data(),
                           msa::kBwdChunk);
          for (int s = 0; s < cnt; ++s)
            for (int c = 0; c < d; ++c) {
              float gk, gv;
              msa::bwd_kv_cols(u, P.data(), dS.data(), msa::kBwdChunk, s, c, &gk, &gv);
              dk_seq[(tok[s] * G + g) * d + c] += gk;
              dv_seq[(tok[s] * G + g) * d + c] += gv;
            }
          for (int h = 0; h < Hg; ++h)
            for (int c0_ = 0; c0_ < d; c0_ += 8)
              msa::bwd_phase2(u, dS.data(), kst.data(), rw, cnt, h, c0_, acc.data() + h * d + c0_);
        }
        for (int o = 0; o < Hg * d; ++o) dq[row0 + o] = sm * acc[o];
      }
    }
  }
  FILE* o = fopen(argv[2], "wb");
  if (!o) return 2;
  fwrite(dq.data(), 4, dq.size(), o);
  fwrite(dk.data(), 4, dk.size(), o);
  fwrite(dv.data(), 4, dv.size(), o);
  fclose(o);
  printf("bad %d\n", bad_total);
  return 0;
}
