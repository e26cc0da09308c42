// Index Branch, decode shape (one query per sequence): block scores over the
// whole index-key cache, then top-(k-1) plus the forced local block
// (pnsm.cn explainer sec. 2, sec. 7 "exp-free Top-k", sec. 9 decoding; yhxrc.cn
// sec. 二).
//
// The step is bound by HBM: every cached index key (d_idx bf16) is read once.
//   scan   : a CTA takes CB consecutive 128-key tiles of one sequence; TMA
//            brings each [128 x d_idx] tile into swizzled shared memory; one
//            warp per tile computes the 128 x G scores with mma.sync (bf16 in,
//            fp32 out; the G index-query heads padded to n = 8) and max-pools
//            them per block of B_k keys (128 / B_k blocks per tile).
//   select : one CTA per (sequence, group): per-thread top-(k-1) over a strided
//            slice of the block scores, then k-1 rounds of block-wide argmax on
//            64-bit keys (score, then lower block index).
#include <climits>

#include "msa_common.cuh"

namespace msa {
namespace {

constexpr int kCB = 4;            // blocks per scan CTA (one warp each)
constexpr int kScanThreads = 32 * kCB;
constexpr int kSelThreads = 256;

size_t scratch_layout(int32_t batch, int64_t total_k, int32_t G, int32_t B_k, size_t* bscore_off,
                      size_t* blk_off_off, size_t* chunk_off_off) {
  const int64_t nblocks = (total_k + B_k - 1) / B_k + batch;
  size_t off = 0;
  *bscore_off = off;
  off = align_up(off + sizeof(float) * nblocks * G, 256);
  *blk_off_off = off;
  off = align_up(off + sizeof(int32_t) * (batch + 1), 256);
  *chunk_off_off = off;
  off = align_up(off + sizeof(int32_t) * (batch + 1), 256);
  return off;
}

// blk_off[b]: first block id of sequence b; chunk_off[b]: first scan chunk.
__global__ void decode_prep_kernel(const int32_t* __restrict__ cu_q, const int32_t* __restrict__ cu_k, int batch,
                                   int B_k, int all_blocks, int32_t* __restrict__ blk_off,
                                   int32_t* __restrict__ chunk_off, DevError* err) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int bo = 0, co = 0;
  for (int b = 0; b < batch; ++b) {
    blk_off[b] = bo;
    chunk_off[b] = co;
    const int Tb = cu_q[b + 1] - cu_q[b];
    const int Sb = cu_k[b + 1] - cu_k[b];
    if (Tb < 0 || Tb > 1 || Tb > Sb) {
      report_error(err, MSA_ERR_DEVICE_CHECK, kSiteDecodeIndex, b, Tb);
    } else if (Tb == 1) {
      // blocks scored: those before the query's local block, or (all_blocks)
      // every complete block of the keys when the query lies after them
      const int lb = all_blocks ? Sb / B_k : (Sb - 1) / B_k;
      const int ntile = (lb * B_k + kBk - 1) / kBk;   // 128-key tiles holding them
      co += (ntile + kCB - 1) / kCB;
    }
    bo += (Sb + B_k - 1) / B_k;
  }
  blk_off[batch] = bo;
  chunk_off[batch] = co;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& a0, uint32_t& a1, uint32_t& a2, uint32_t& a3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int DIDX>
__global__ void __launch_bounds__(kScanThreads)
decode_scan_kernel(const __grid_constant__ CUtensorMap tm_k, const __nv_bfloat16* __restrict__ q_idx,
                   const int32_t* __restrict__ cu_q, const int32_t* __restrict__ cu_k, int batch, int G, int B_k,
                   int all_blocks,
                   const int32_t* __restrict__ blk_off, const int32_t* __restrict__ chunk_off,
                   float* __restrict__ bscore, const int32_t* __restrict__ block_table, int max_blocks,
                   int64_t num_pages, DevError* err) {
  constexpr int SPAN = DIDX * 2 >= 128 ? 128 : DIDX * 2;
  constexpr int NBOX = DIDX * 2 / SPAN;
  constexpr int BLOCK_BYTES = kBk * DIDX * 2;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kCB * BLOCK_BYTES);

  const int chunk = blockIdx.x;
  if (chunk >= chunk_off[batch]) return;
  // sequence of this chunk: the last b with chunk_off[b] <= chunk (sequences
  // without chunks share their offset with the next one)
  int lo = 0, hi = batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (chunk_off[mid] <= chunk) lo = mid; else hi = mid;
  }
  const int b = lo;
  const int Sb = cu_k[b + 1] - cu_k[b];
  const int lb = all_blocks ? Sb / B_k : (Sb - 1) / B_k;   // blocks scored: 0 .. lb - 1
  const int ntile = (lb * B_k + kBk - 1) / kBk;     // 128-key tiles holding them
  const int bpt = kBk / B_k;                        // blocks per tile
  const int j0 = (chunk - chunk_off[b]) * kCB;      // first tile of this chunk
  const int nblk = min(kCB, ntile - j0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // first key row of block j0 + i (packed: after the sequence's start; paged:
  // its page); -1: an invalid page, whose block is not read
  auto block_row = [&](int i) -> int64_t {
    if (block_table == nullptr) return (int64_t)cu_k[b] + (int64_t)kBk * (j0 + i);
    const int32_t pg = block_table[(int64_t)b * max_blocks + j0 + i];
    return (pg >= 0 && pg < num_pages) ? (int64_t)pg * kBk : -1;
  };
  if (threadIdx.x == 0) {
    for (int i = 0; i < kCB; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    for (int i = 0; i < nblk; ++i) {
      const int64_t row = block_row(i);
      if (row < 0) {
        report_error(err, MSA_ERR_DEVICE_CHECK, kSitePaged, b, j0 + i);
        continue;
      }
      mbar_arrive_expect_tx(&bars[i], BLOCK_BYTES);
      for (int bx = 0; bx < NBOX; ++bx)
        tma_load_2d(smem + i * BLOCK_BYTES + bx * kBk * SPAN, &tm_k, &bars[i], bx * (SPAN / 2), (int)row);
    }
  }
  // B operand: q_idx of this sequence's query, n = group (zero for n >= G).
  const int64_t qrow = cu_q[b];
  const int n = lane >> 2;
  uint32_t bfrag[DIDX / 16][2];
#pragma unroll
  for (int kk = 0; kk < DIDX / 16; ++kk) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int kidx = kk * 16 + 2 * (lane & 3) + 8 * h;
      uint32_t v = 0;
      if (n < G) v = *reinterpret_cast<const uint32_t*>(q_idx + (qrow * G + n) * DIDX + kidx);
      bfrag[kk][h] = v;
    }
  }
  __syncthreads();
  if (warp < nblk && block_row(warp) < 0) {
    // an invalid page: the block was not read and ranks last
    if (lane < G) bscore[(int64_t)(blk_off[b] + j0 + warp) * G + lane] = -INFINITY;
  } else if (warp < nblk) {
    if (!mbar_wait(&bars[warp], 0)) {
      report_error(err, MSA_ERR_TIMEOUT, kSiteDecodeIndex, chunk, warp);
    } else {
      const uint32_t base = smem_u32(smem + warp * BLOCK_BYTES);
      const int mt_per_blk = B_k / 16;                 // 16-row MMA tiles per block
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll 2
      for (int mt = 0; mt < kBk / 16; ++mt) {
        float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < DIDX / 16; ++kk) {
          const int r = 16 * mt + (lane & 15);
          const int chunk16 = 2 * kk + (lane >> 4);          // 16-byte chunk along d_idx
          const int box = (chunk16 * 16) / SPAN;
          const int cin = chunk16 % (SPAN / 16);
          const uint32_t addr = base + box * (kBk * SPAN) + swz_offset(r, cin, SPAN);
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4(addr, a0, a1, a2, a3);
          mma_bf16_16816(c, a0, a1, a2, a3, bfrag[kk][0], bfrag[kk][1]);
        }
        mx0 = fmaxf(mx0, fmaxf(c[0], c[2]));
        mx1 = fmaxf(mx1, fmaxf(c[1], c[3]));
        if ((mt + 1) % mt_per_blk == 0) {
          // the last rows of block (tile j0 + warp) * bpt + mt / mt_per_blk
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
          }
          const int blk = (j0 + warp) * bpt + mt / mt_per_blk;
          if (lane < 4 && blk < lb) {
            const int64_t gb = (int64_t)(blk_off[b] + blk) * G;
            const int g0 = 2 * lane, g1 = 2 * lane + 1;
            if (g0 < G) bscore[gb + g0] = (mx0 != mx0) ? -INFINITY : mx0;
            if (g1 < G) bscore[gb + g1] = (mx1 != mx1) ? -INFINITY : mx1;
          }
          mx0 = -INFINITY;
          mx1 = -INFINITY;
        }
      }
    }
  }
  // no load may remain in flight when the CTA exits
  if (threadIdx.x == 0)
    for (int i = 0; i < nblk; ++i)
      if (block_row(i) >= 0) mbar_wait(&bars[i], 0);
}

// Paged decode: logical offsets of one query per sequence and its cache.
__global__ void paged_prep_kernel(const int32_t* __restrict__ seqlens, int batch, int max_blocks,
                                  int32_t* __restrict__ cu_q, int32_t* __restrict__ cu_k, DevError* err) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int64_t acc = 0;
  for (int b = 0; b < batch; ++b) {
    cu_q[b] = b;
    cu_k[b] = (int32_t)acc;
    int32_t L = seqlens[b];
    if (L < 1 || (int64_t)L > (int64_t)max_blocks * kBk || acc + L > INT32_MAX) {
      report_error(err, MSA_ERR_DEVICE_CHECK, kSitePaged, b, L);
      L = 0;                                   // the sequence then takes no part
    }
    acc += L;
  }
  cu_q[batch] = batch;
  cu_k[batch] = (int32_t)acc;
}

// 64-bit ranking key: order-preserving score bits, then the complement of the
// block id (lower id ranks higher).  Real keys are > 0; 0 marks an empty slot.
__device__ __forceinline__ uint64_t rank_key(float s, int j) {
  uint32_t u = __float_as_uint(s);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<uint64_t>(u) << 32) | static_cast<uint32_t>(~j);
}

// kCand == false: the selection (best k-1 earlier blocks, then the forced
// local block; ascending ids, -1 padding).  kCand == true: the candidates of a
// key range (the best k-1 of the scored blocks in rank order, with their
// scores; -1 / -inf padding), for a selection merged over several ranges.
template <int CAP, bool kCand>
__global__ void __launch_bounds__(kSelThreads)
decode_select_kernel(const float* __restrict__ bscore, const int32_t* __restrict__ cu_q,
                     const int32_t* __restrict__ cu_k, const int32_t* __restrict__ blk_off, int G, int k, int B_k,
                     int all_blocks, int32_t* __restrict__ sel, float* __restrict__ cand_score) {
  const int b = blockIdx.x / G, g = blockIdx.x % G;
  const int Tb = cu_q[b + 1] - cu_q[b];
  const int Sb = cu_k[b + 1] - cu_k[b];
  const int width = kCand ? k - 1 : k;   // output entries per (query, group)
  if (Tb == 1 && Sb < 1) {
    // a query without keys (an error the prep recorded): an empty selection
    if (threadIdx.x < width) {
      sel[((int64_t)cu_q[b] * G + g) * width + threadIdx.x] = -1;
      if (kCand) cand_score[((int64_t)cu_q[b] * G + g) * width + threadIdx.x] = -INFINITY;
    }
    return;
  }
  if (Tb != 1) return;
  const int lb = all_blocks ? Sb / B_k : (Sb - 1) / B_k;
  const int cap = k - 1;
  const float* sc = bscore + (int64_t)blk_off[b] * G + g;
  // per-thread sorted (descending) list of the best keys of its slice
  uint64_t list[CAP];
#pragma unroll
  for (int i = 0; i < CAP; ++i) list[i] = 0;
  // (the list keeps CAP >= k-1 entries; the merge below takes the global best)
  for (int j = threadIdx.x; j < lb; j += kSelThreads) {
    const uint64_t key = rank_key(sc[(int64_t)j * G], j);
    if (key > list[CAP - 1]) {
#pragma unroll
      for (int i = CAP - 1; i >= 1; --i) {
        const bool gt_prev = key > list[i - 1];
        const bool gt_here = key > list[i];
        list[i] = gt_prev ? list[i - 1] : (gt_here ? key : list[i]);
      }
      if (key > list[0]) list[0] = key;
    }
  }
  // k-1 rounds of block-wide argmax over the list heads
  __shared__ uint64_t warp_best[kSelThreads / 32];
  __shared__ int32_t chosen[kMaxK];
  __shared__ float chosen_score[kMaxK];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nsel = min(cap, lb);
  for (int r = 0; r < nsel; ++r) {
    uint64_t best = list[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint64_t other = __shfl_xor_sync(0xffffffffu, best, o);
      best = other > best ? other : best;
    }
    if (lane == 0) warp_best[wid] = best;
    __syncthreads();
    uint64_t top = 0;
#pragma unroll
    for (int w = 0; w < kSelThreads / 32; ++w) top = warp_best[w] > top ? warp_best[w] : top;
    if (list[0] == top && top != 0) {   // keys are unique: one owner pops its head
#pragma unroll
      for (int i = 0; i < CAP - 1; ++i) list[i] = list[i + 1];
      list[CAP - 1] = 0;
    }
    if (threadIdx.x == 0) {
      chosen[r] = (int)~static_cast<uint32_t>(top & 0xffffffffu);
      // the key's upper half holds the order-preserving score bits
      uint32_t u = static_cast<uint32_t>(top >> 32);
      u = (u & 0x80000000u) ? (u & 0x7fffffffu) : ~u;
      chosen_score[r] = __uint_as_float(u);
    }
    __syncthreads();
  }
  if (kCand) {
    // candidates in the order chosen (score descending, lower id first)
    if (threadIdx.x < width) {
      const int64_t o = ((int64_t)cu_q[b] * G + g) * width + threadIdx.x;
      sel[o] = threadIdx.x < nsel ? chosen[threadIdx.x] : -1;
      cand_score[o] = threadIdx.x < nsel ? chosen_score[threadIdx.x] : -INFINITY;
    }
    return;
  }
  if (threadIdx.x == 0) {
    // ascending ids, then the local block, then -1
    for (int i = 1; i < nsel; ++i) {
      const int v = chosen[i];
      int p = i - 1;
      while (p >= 0 && chosen[p] > v) { chosen[p + 1] = chosen[p]; --p; }
      chosen[p + 1] = v;
    }
    int32_t* dst = sel + ((int64_t)cu_q[b] * G + g) * k;
    for (int i = 0; i < nsel; ++i) dst[i] = chosen[i];
    dst[nsel] = lb;
    for (int i = nsel + 1; i < k; ++i) dst[i] = -1;
  }
}

}  // namespace

size_t decode_index_scratch_bytes(int32_t batch, int64_t total_k, int32_t G, int32_t B_k) {
  size_t a, b, c;
  return scratch_layout(batch, total_k, G, B_k, &a, &b, &c);
}

int launch_index_topk_decode(const IndexTopkArgs& a, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  size_t o_bs, o_bo, o_co;
  const size_t need = scratch_layout(a.batch, a.total_k, a.G, a.B_k, &o_bs, &o_bo, &o_co);
  if (a.scratch_bytes < need) return (int)cudaErrorInvalidValue;
  uint8_t* base = static_cast<uint8_t*>(a.scratch);
  float* bscore = reinterpret_cast<float*>(base + o_bs);
  int32_t* blk_off = reinterpret_cast<int32_t*>(base + o_bo);
  int32_t* chunk_off = reinterpret_cast<int32_t*>(base + o_co);
  {
    ProfScope p("decode_prep", stream);
    decode_prep_kernel<<<1, 32, 0, st>>>(a.cu_q, a.cu_k, a.batch, a.B_k, a.all_blocks, blk_off, chunk_off, a.err);
  }

  const int span = a.d_idx * 2 >= 128 ? 128 : a.d_idx * 2;
  alignas(64) CUtensorMap tm_k;
  const uint64_t rows = a.block_table != nullptr ? (uint64_t)a.num_pages * kBk : (uint64_t)a.total_k;
  const uint64_t dims[2] = {(uint64_t)a.d_idx, rows};
  const uint64_t strides[1] = {(uint64_t)a.d_idx * 2};
  const uint32_t box[2] = {(uint32_t)(span / 2), (uint32_t)kBk};
  int rc = make_tmap_bf16(&tm_k, a.k_idx, 2, dims, strides, box, span);
  if (rc) return rc;
  // upper bound of scan chunks; the kernel drops the surplus
  const int64_t max_chunks = (a.total_k + (int64_t)kBk * kCB - 1) / ((int64_t)kBk * kCB) + a.batch;
  const size_t smem = 1024 + (size_t)kCB * kBk * a.d_idx * 2 + 64;
  const __nv_bfloat16* qi = reinterpret_cast<const __nv_bfloat16*>(a.q_idx);
  cudaError_t e;
#define MSA_SCAN(D)                                                                                          \
  e = cudaFuncSetAttribute(decode_scan_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);  \
  if (e != cudaSuccess) return (int)e;                                                                      \
  ProfScope p("decode_scan", stream);                                                                       \
  decode_scan_kernel<D><<<(unsigned)max_chunks, kScanThreads, smem, st>>>(                                  \
      tm_k, qi, a.cu_q, a.cu_k, a.batch, a.G, a.B_k, a.all_blocks, blk_off, chunk_off, bscore, a.block_table,  \
      a.max_blocks,                                                                                          \
      a.num_pages, a.err)
  if (a.d_idx == 32) { MSA_SCAN(32); }
  else if (a.d_idx == 64) { MSA_SCAN(64); }
  else { MSA_SCAN(128); }
#undef MSA_SCAN
  const unsigned nsel = (unsigned)(a.batch * a.G);
  ProfScope p("decode_select", stream);
#define MSA_SEL(CAP)                                                                                         \
  if (a.cand_score != nullptr)                                                                               \
    decode_select_kernel<CAP, true><<<nsel, kSelThreads, 0, st>>>(bscore, a.cu_q, a.cu_k, blk_off, a.G, a.k,  \
                                                                 a.B_k, a.all_blocks, a.sel, a.cand_score);  \
  else                                                                                                       \
    decode_select_kernel<CAP, false><<<nsel, kSelThreads, 0, st>>>(bscore, a.cu_q, a.cu_k, blk_off, a.G, a.k, \
                                                                  a.B_k, a.all_blocks, a.sel, nullptr);
  if (a.k <= 8) { MSA_SEL(7) }
  else if (a.k <= 16) { MSA_SEL(15) }
  else { MSA_SEL(31) }
#undef MSA_SEL
  return (int)cudaGetLastError();
}

int launch_paged_prep(const int32_t* seqlens, int32_t batch, int32_t max_blocks, int32_t* cu_q, int32_t* cu_k,
                      DevError* err, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope p("paged_prep", stream);
  paged_prep_kernel<<<1, 32, 0, st>>>(seqlens, batch, max_blocks, cu_q, cu_k, err);
  return (int)cudaGetLastError();
}

}  // namespace msa
