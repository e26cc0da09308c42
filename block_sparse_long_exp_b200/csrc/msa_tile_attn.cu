// Main Branch, query-tile side (Q-outer), and dense causal GQA.
//
// The pages' KV-outer schedule (pnsm.cn explainer sec. 7 "KV-outer sparse
// attention", "two-phase combine") writes one normalised partial per
// (query, group, selected block) and merges them afterwards.  With Hg = 16
// heads of d = 128 a partial is 4 KB of f16 against ~1 MFLOP of tensor-core
// work, so on B200 the partials' round trip through HBM costs more time than
// the attention arithmetic.  Neighbouring queries often select the same
// blocks (every query keeps its local block, and hot blocks attract most
// queries), so the blocks that many queries of a small query tile share are
// attended here instead, query-tile-major: the tile's Q rows stay in shared
// memory, the shared blocks stream through, and an online softmax (running
// max / sum per row, O accumulated in TMEM) merges them into ONE result per
// query.  A query whose every selection is covered writes its final output
// directly; otherwise its merged result becomes one partial for the combine,
// and its remaining selections go through the KV-outer lists.  The result is
// the same exact softmax over the same selected token set (the merge order of
// the blocks differs, which changes only rounding).
//
// Units: a tile of UQ = 2 x (128 / RQ) consecutive query rows of one sequence
// (two 128-row MMA tiles of 128 / RQ queries x RQ head rows) and one group.
//
// tile_plan_kernel   one warp per (unit, group): sorts the unit's selections,
//                    keeps the blocks chosen by >= theta of its queries (the
//                    unit's dense blocks, ascending), and per query the slot
//                    mask of those selections, their positions in the dense
//                    list, whether they cover the query, and the combine
//                    list: each query that still needs the combine with its
//                    number of partials (packed at the front of its slot run:
//                    the tile's merged partial first, then the KV-outer ones).
// tile_attn_kernel   persistent, warp-specialised (one CTA per SM, 512 threads):
//   warp 0      claims units (atomic ticket) and publishes them in a 2-deep
//               shared-memory ring;
//   warp 1      owns TMEM (512 columns: per MMA tile 128 columns S/P + d columns
//               O); its lane 0 issues every MMA (S = Q K^T and O += P V of both
//               tiles, interleaved; warp 2 is idle);
//   warp 3      lane 0 TMA-loads the unit's Q tiles and every K / V block
//               (two stages);
//   warps 4-7   online softmax of MMA tile 0, warps 8-11 of MMA tile 1: S -> P
//               (bf16, into the S columns), running max / sum per row; when a
//               row's max grows by more than 2^8 the O row is rescaled in TMEM
//               (only then);
//   warps 12-15 epilogue: O / l -> bf16 output (or an f16 partial) and the
//               log-sum-exp.
// In dense mode a unit's blocks are 0 .. the last query's block and a row
// attends every key at or before its position: dense causal GQA, the baseline
// of the pages' speedup comparison (pnsm.cn sec. 9).  In rows mode a unit is
// one query and its selection row (decode: one query per sequence), written
// straight to the output.
#include <climits>

#include "msa_common.cuh"

namespace msa {
namespace {

constexpr int kTileThreads = 512;
constexpr int kUnitRing = 2;
constexpr int kUnitEmptyCount = 14;      // MMA issuer, loader, 8 softmax warps, 4 epilogue warps
constexpr float kRescaleLog2 = 8.f;      // rescale O only when the row max grows by more than 2^8
constexpr int kPlanWarps = 4;

// What a unit is (template argument of tile_attn_kernel):
//   kModeTiles  a tile of UQ queries and its dense blocks (tile_plan_kernel);
//   kModeDense  a tile of UQ queries and every block up to its last query
//               (dense causal GQA);
//   kModeRows   one query and the blocks of its selection row (decode: the
//               Q-outer form of a single query, no partials).
constexpr int kModeTiles = 0, kModeDense = 1, kModeRows = 2;
constexpr int kPlanMaxEntries = 1024;    // UQ x k <= 32 x 32

__device__ __forceinline__ int find_seq_t(const int32_t* __restrict__ cu, int batch, int64_t row) {
  int lo = 0, hi = batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu[mid] <= row) lo = mid; else hi = mid;
  }
  return lo;
}

// ------------------------------------------------------------- planner ---

__global__ void __launch_bounds__(kPlanWarps * 32)
tile_plan_kernel(const int32_t* __restrict__ sel, int64_t t0, int64_t t1, int G, int k, int UQ, int theta,
                 int batch, const int32_t* __restrict__ cu_q, int32_t* __restrict__ unit_blk,
                 int32_t* __restrict__ unit_nblk, int32_t* __restrict__ unit_list, uint32_t* __restrict__ dmask,
                 int32_t* __restrict__ dstate, uint64_t* __restrict__ dmember, uint2* __restrict__ clist,
                 int32_t* __restrict__ counters) {
  __shared__ int32_t s_vals[kPlanWarps][kPlanMaxEntries];
  __shared__ int32_t s_dense[kPlanWarps][kMaxDense];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nunits = (t1 - t0 + UQ - 1) / UQ;
  const int64_t w = (int64_t)blockIdx.x * kPlanWarps + warp;
  if (w >= nunits * G) return;                 // whole warps only; no block-wide barrier below
  const int64_t unit = w / G;
  const int g = (int)(w - unit * G);
  const int64_t r0 = t0 + unit * UQ;
  const int nq = (int)(t1 - r0 < UQ ? t1 - r0 : UQ);
  const bool one_seq = find_seq_t(cu_q, batch, r0) == find_seq_t(cu_q, batch, r0 + nq - 1);
  const int n = UQ * k;
  int NS = 1;
  while (NS < n) NS <<= 1;
  int32_t* v = s_vals[warp];
  for (int i = lane; i < NS; i += 32) {
    int32_t x = INT_MAX;
    if (i < n) {
      const int q = i / k, s = i - q * k;
      if (one_seq && q < nq) {
        const int32_t b = sel[((r0 + q) * G + g) * k + s];
        if (b >= 0) x = b;
      }
    }
    v[i] = x;
  }
  __syncwarp();
  // bitonic sort, ascending (unused entries are INT_MAX and sort last)
  for (int size = 2; size <= NS; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = lane; i < NS / 2; i += 32) {
        const int lo = 2 * stride * (i / stride) + (i % stride), hi = lo + stride;
        const bool up = (lo & size) == 0;
        const int32_t a = v[lo], b = v[hi];
        if ((a > b) == up) { v[lo] = b; v[hi] = a; }
      }
      __syncwarp();
    }
  }
  // runs of at least theta equal block ids, in ascending order, at most kMaxDense
  int nd = 0;
  for (int base = 0; base < NS && nd < kMaxDense; base += 32) {
    const int i = base + lane;
    bool take = false;
    int32_t x = INT_MAX;
    if (i < NS) {
      x = v[i];
      if (x != INT_MAX && (i == 0 || v[i - 1] != x)) {
        int c = 1;
        while (c < theta && i + c < NS && v[i + c] == x) ++c;
        take = c >= theta;
      }
    }
    const unsigned bal = __ballot_sync(0xffffffffu, take);
    const int p = nd + __popc(bal & ((1u << lane) - 1u));
    if (take && p < kMaxDense) s_dense[warp][p] = x;
    nd += __popc(bal);
  }
  if (nd > kMaxDense) nd = kMaxDense;
  __syncwarp();
  // lane q: masks of query q (UQ <= 32)
  const bool qv = lane < nq;
  bool need_combine = false;
  uint32_t cmask = 0;                          // number of packed partials to merge
  if (qv) {
    const int64_t t = r0 + lane;
    uint32_t dm = 0, vm = 0;
    uint64_t mem = 0;
    for (int s = 0; s < k; ++s) {
      const int32_t b = sel[(t * G + g) * k + s];
      if (b < 0) continue;
      vm |= 1u << s;
      int lo = 0, hi = nd;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (s_dense[warp][mid] < b) lo = mid + 1; else hi = mid;
      }
      if (lo < nd && s_dense[warp][lo] == b) {
        dm |= 1u << s;
        mem |= 1ull << lo;
      }
    }
    const int64_t pr = (t - t0) * G + g;
    const bool complete = dm != 0 && dm == vm;
    dmask[pr] = dm;
    dmember[pr] = mem;
    dstate[pr] = dm == 0 ? -1 : (complete ? kDenseComplete : 0);
    need_combine = !complete;
    cmask = (uint32_t)__popc(vm & ~dm) + (dm != 0u ? 1u : 0u);   // packed: the tile's, then the KV-outer ones
  }
  const unsigned bal = __ballot_sync(0xffffffffu, need_combine);
  int base = 0;
  if (lane == 0 && bal != 0u) base = atomicAdd(&counters[0], __popc(bal));
  base = __shfl_sync(0xffffffffu, base, 0);
  if (need_combine)
    clist[base + __popc(bal & ((1u << lane) - 1u))] = make_uint2((uint32_t)((r0 + lane - t0) * G + g), cmask);
  if (lane == 0) unit_nblk[w] = nd;
  for (int j = lane; j < nd; j += 32) unit_blk[w * kMaxDense + j] = s_dense[warp][j];
  if (lane == 0 && nd > 0) unit_list[atomicAdd(&counters[1], 1)] = (int32_t)w;
}

// Dense mode: units per sequence (prefix over the batch) and their total.
__global__ void dense_units_kernel(const int32_t* __restrict__ cu_q, int batch, int UQ, int G,
                                   int32_t* __restrict__ seq_units, int32_t* __restrict__ counters) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    int acc = 0;
    for (int b = 0; b < batch; ++b) {
      seq_units[b] = acc;
      acc += (cu_q[b + 1] - cu_q[b] + UQ - 1) / UQ;
    }
    seq_units[batch] = acc;
    counters[1] = acc * G;
    counters[2] = 0;
  }
}

// ----------------------------------------------------- tile attention ---

struct __align__(16) TileUnit {
  int64_t r0;                 // first query row (absolute)
  int32_t uid, g, nq, nblk;   // nblk < 0: no more work
  int32_t ntl, Tb, Sb, qrow0;
  int32_t kbase, pad0, pad1, pad2;
  int32_t blk[kMaxDense];     // tiles / rows mode: the unit's blocks, ascending
  int32_t page[kMaxDense];    // rows mode with a page table: each block's page
};

struct __align__(16) TileCtl {
  uint64_t unit_full[kUnitRing], unit_empty[kUnitRing];
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[2], v_full[2], kv_empty[2];
  uint64_t s_full[2], p_half[2], p_full[2], pv_done[2], o_free[2], stats_full[2];
  uint64_t mma_done[2];
  uint32_t tmem_base;
  int32_t abort_flag;
  int32_t pad[2];
  TileUnit ring[kUnitRing];
  float row_m[2][128];        // final running max (log2 units) per row, per MMA tile
  float row_l[2][128];        // final running sum per row, per MMA tile
};

struct TileParams {
  const int32_t* unit_list;   // hybrid: units with dense blocks
  const int32_t* unit_blk;    // hybrid: [units x G][kMaxDense]
  const int32_t* unit_nblk;
  const uint64_t* dmember;    // hybrid: [rows x G] dense-list membership bits
  const int32_t* dstate;      // tiles mode: [rows x G] -1 none covered, 0 some, kDenseComplete all
  const int32_t* seq_units;   // dense: [batch + 1] prefix of units per sequence
  const int32_t* nunits;      // device count of units (tiles: listed units; dense: all); null: nunits_host
  int64_t nunits_host;        // rows mode: rows x G
  const int32_t* sel;         // rows mode: [T, G, k]
  const int32_t* block_table; // rows mode, paged caches: [batch, max_blocks] page per block (else null)
  int32_t max_blocks;
  int64_t num_pages;
  int32_t* ticket;
  const int32_t* cu_q;
  const int32_t* cu_k;
  int32_t batch, H, G, d, k, UQ;
  int32_t bk;                 // block size B_k (tiles and rows modes; dense mode works in 128-key tiles)
  float scale_log2;
  int64_t t0, t1;
  __nv_bfloat16* out;         // [T, H, d] (absolute rows)
  float* lse;                 // [T, H] or null
  __half* part_acc;           // hybrid: partials of the pass (rows relative to t0)
  float* part_lse;
  DevError* err;
};

template <int kMode>
__global__ void __launch_bounds__(kTileThreads, 1)
tile_attn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ TileParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int d = p.d;
  const int tile_bytes = 128 * d * 2;         // one [128 x d] bf16 tile
  uint8_t* kv_s = smem;                        // 2 stages x (K, V)
  uint8_t* q_s = kv_s + 4 * tile_bytes;        // 2 MMA tiles of Q
  TileCtl* ctl = reinterpret_cast<TileCtl*>(q_s + 2 * tile_bytes);
  volatile int32_t* abort_flag = &ctl->abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.G, H = p.H, Hg = H / G;
  const int RQ = Hg < 8 ? 8 : Hg;              // tile rows per query
  const int qpt = 128 / RQ;                    // queries per MMA tile
  const int nhalf = d / 64;

  if (tid == 0) {
    for (int i = 0; i < kUnitRing; ++i) {
      mbar_init(&ctl->unit_full[i], 1);
      mbar_init(&ctl->unit_empty[i], kUnitEmptyCount);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->q_full[i], 1); mbar_init(&ctl->q_empty[i], 1);
      mbar_init(&ctl->k_full[i], 1); mbar_init(&ctl->v_full[i], 1); mbar_init(&ctl->kv_empty[i], 1);
      mbar_init(&ctl->s_full[i], 1); mbar_init(&ctl->p_half[i], 4); mbar_init(&ctl->p_full[i], 4);
      mbar_init(&ctl->pv_done[i], 1); mbar_init(&ctl->o_free[i], 4);
      mbar_init(&ctl->stats_full[i], 4);
      mbar_init(&ctl->mma_done[i], 1);
    }
    ctl->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_q);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  auto wait_unit = [&](int n) -> const TileUnit* {
    const int slot = n % kUnitRing;
    if (!mbar_wait(&ctl->unit_full[slot], (n / kUnitRing) & 1)) {
      report_error(p.err, MSA_ERR_TIMEOUT, kSiteTileUnit, n, warp);
      *abort_flag = 1;
      return nullptr;
    }
    return &ctl->ring[slot];
  };
  auto release_unit = [&](int n, bool whole_warp) {
    if (whole_warp) __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->unit_empty[n % kUnitRing]);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ scheduler
    const int64_t nun = p.nunits != nullptr ? (int64_t)*p.nunits : p.nunits_host;
    int n = 0;
    while (true) {
      const int slot = n % kUnitRing;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&ctl->unit_empty[slot], ((n / kUnitRing) + 1) & 1);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) {
        if (lane == 0) report_error(p.err, MSA_ERR_TIMEOUT, kSiteTileUnit, n, -1);
        *abort_flag = 1;
        break;
      }
      int64_t it = 0;
      if (lane == 0) it = *abort_flag ? nun : (int64_t)atomicAdd(p.ticket, 1);
      it = __shfl_sync(0xffffffffu, it, 0);
      TileUnit* U = &ctl->ring[slot];
      if (it >= nun) {
        if (lane == 0) {
          U->nblk = -1;
          mbar_arrive(&ctl->unit_full[slot]);
        }
        break;
      }
      int32_t uid, g, nq, nblk, seq;
      int64_t r0;
      if (kMode == kModeRows) {
        const int64_t t = p.t0 + it / G;
        g = (int)(it - (t - p.t0) * G);
        r0 = t;
        nq = 1;
        seq = find_seq_t(p.cu_q, p.batch, r0);
        uid = (int32_t)it;
      } else if (kMode == kModeDense) {
        // longest units first: reverse order (the last tiles of a sequence see the most blocks)
        const int64_t v = nun - 1 - it;
        const int64_t tg = v / G;
        g = (int)(v - tg * G);
        int lo = 0, hi = p.batch;
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (p.seq_units[mid] <= tg) lo = mid; else hi = mid;
        }
        seq = lo;
        r0 = p.cu_q[seq] + (tg - p.seq_units[seq]) * p.UQ;
        const int64_t rend = p.cu_q[seq + 1];
        nq = (int)(rend - r0 < p.UQ ? rend - r0 : p.UQ);
        uid = (int32_t)v;
      } else {
        uid = p.unit_list[it];
        const int64_t unit = uid / G;
        g = uid - (int32_t)unit * G;
        r0 = p.t0 + unit * p.UQ;
        nq = (int)(p.t1 - r0 < p.UQ ? p.t1 - r0 : p.UQ);
        seq = find_seq_t(p.cu_q, p.batch, r0);
      }
      const int Tb = p.cu_q[seq + 1] - p.cu_q[seq];
      const int Sb = p.cu_k[seq + 1] - p.cu_k[seq];
      if (kMode == kModeRows) {
        // the selection row: valid ids first, then -1 padding; a row with an
        // id past the query's block (or a page outside the cache) is reported
        // and skipped before anything is read
        const int32_t b = lane < p.k ? p.sel[(r0 * G + g) * p.k + lane] : -1;
        const unsigned v = __ballot_sync(0xffffffffu, b >= 0);
        nblk = __popc(v);
        const int64_t pos = (int64_t)Sb - Tb + (r0 - p.cu_q[seq]);
        bool bad = b >= 0 && (Tb > Sb || pos < 0 || b > pos / p.bk);
        int32_t pg = -1;
        if (b >= 0 && !bad && p.block_table != nullptr) {
          bad = b >= p.max_blocks;
          if (!bad) {
            pg = p.block_table[(int64_t)seq * p.max_blocks + b];
            bad = pg < 0 || pg >= p.num_pages;
          }
        }
        if (bad) report_error(p.err, MSA_ERR_DEVICE_CHECK, p.block_table != nullptr ? kSitePaged : kSiteInvert,
                              (int)r0, b);
        if (b >= 0) {
          U->blk[lane] = b;
          U->page[lane] = pg;
        }
        const bool any_bad = __any_sync(0xffffffffu, bad);
        if (any_bad || v != (nblk >= 32 ? 0xffffffffu : (1u << nblk) - 1u)) {
          // ids must come first: anything else is not a selection row
          if (lane == 0 && !any_bad) report_error(p.err, MSA_ERR_DEVICE_CHECK, kSiteInvert, (int)r0, -1);
          nblk = 0;
        }
      } else if (kMode == kModeDense) {
        const int64_t pos_last = (int64_t)Sb - Tb + (r0 + nq - 1 - p.cu_q[seq]);
        nblk = (int)(pos_last / kBk) + 1;
        if (Tb > Sb) {
          if (lane == 0) report_error(p.err, MSA_ERR_DEVICE_CHECK, kSiteDense, seq, Tb);
          nblk = 0;
        }
      } else {
        nblk = p.unit_nblk[uid];
        if (nblk > kMaxDense) nblk = kMaxDense;
        for (int j = lane; j < nblk; j += 32) U->blk[j] = p.unit_blk[(int64_t)uid * kMaxDense + j];
      }
      if (lane == 0) {
        U->r0 = r0; U->uid = uid; U->g = g; U->nq = nq; U->nblk = nblk;
        U->ntl = nblk > 0 ? (nq > qpt ? 2 : 1) : 0;   // no block: no tile takes part
        U->Tb = Tb; U->Sb = Sb; U->qrow0 = p.cu_q[seq]; U->kbase = p.cu_k[seq];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->unit_full[slot]);
      ++n;
    }
  } else if (warp == 3) {
    // --------------------------------------------------------------- loader
    if (lane == 0) {
      int n = 0, uq[2] = {0, 0};
      int64_t kvc = 0;
      bool ok = true;
      while (ok && !*abort_flag) {
        const TileUnit* R = wait_unit(n);
        if (R == nullptr) { ok = false; break; }
        const int nblk = R->nblk;
        if (nblk < 0) break;
        const int ntl = R->ntl, g = R->g;
        const int64_t r0 = R->r0;
        const int kbase = R->kbase;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (x >= ntl || !ok) continue;
          ok = mbar_wait(&ctl->q_empty[x], (uq[x] + 1) & 1);
          if (!ok) continue;
          mbar_arrive_expect_tx(&ctl->q_full[x], tile_bytes);
          for (int h = 0; h < nhalf; ++h)
            tma_load_3d(q_s + x * tile_bytes + h * 128 * 128, &tm_q, &ctl->q_full[x], 64 * h, g * Hg,
                        (int)(r0 + x * qpt));
          ++uq[x];
        }
        for (int j = 0; j < nblk && ok; ++j) {
          const int st = (int)(kvc & 1);
          ok = mbar_wait(&ctl->kv_empty[st], ((kvc >> 1) + 1) & 1);
          if (!ok) break;
          const int blk = kMode == kModeDense ? j : R->blk[j];
          // a block's 128-row K/V tile: B_k rows of it are the block (paged caches: B_k = 128)
          const int krow = (kMode == kModeRows && p.block_table != nullptr) ? R->page[j] * kBk
                         : kbase + blk * (kMode == kModeDense ? kBk : p.bk);
          uint8_t* ks = kv_s + st * 2 * tile_bytes;
          mbar_arrive_expect_tx(&ctl->k_full[st], tile_bytes);
          for (int h = 0; h < nhalf; ++h) tma_load_3d(ks + h * 128 * 128, &tm_k, &ctl->k_full[st], 64 * h, g, krow);
          mbar_arrive_expect_tx(&ctl->v_full[st], tile_bytes);
          for (int h = 0; h < nhalf; ++h)
            tma_load_3d(ks + tile_bytes + h * 128 * 128, &tm_v, &ctl->v_full[st], 64 * h, g, krow);
          ++kvc;
        }
        release_unit(n, false);
        ++n;
      }
      if (!ok) {
        report_error(p.err, MSA_ERR_TIMEOUT, kSiteTileLoad, n, (int)kvc);
        *abort_flag = 1;
      }
      // no TMA load may still be in flight when the CTA exits
      for (int st = 0; st < 2; ++st) {
        const int64_t issued = kvc > st ? (kvc - st + 1) / 2 : 0;
        if (issued > 0) {
          mbar_wait(&ctl->k_full[st], (uint32_t)((issued - 1) & 1));
          mbar_wait(&ctl->v_full[st], (uint32_t)((issued - 1) & 1));
        }
      }
#pragma unroll
      for (int x = 0; x < 2; ++x)
        if (uq[x] > 0) mbar_wait(&ctl->q_full[x], (uq[x] - 1) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // One thread issues every MMA, interleaving the two tiles: S0(j), PV1(j-1),
    // S1(j), PV0(j), S0(j+1), ...  tcgen05.mma operations of one thread run in
    // issue order, so S(j+1) may overwrite the columns that PV(j) reads as P
    // right after PV(j) is issued (no wait for its completion).
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(128, d, 0, 1);
      const uint64_t qdesc0 = make_sdesc(smem_u32(q_s), 16, 1024, kSw128);
      const uint64_t kdesc0 = make_sdesc(smem_u32(kv_s), 16, 1024, kSw128);
      const uint64_t vdesc0 = make_sdesc(smem_u32(kv_s + tile_bytes), 128 * 128, 1024, kSw128);
      int n = 0, ut[2] = {0, 0};
      int64_t kvc = 0, bt[2] = {0, 0};
      bool ok = true;
      auto issue_s = [&](int x, int st) {
        const uint64_t qd = qdesc0 + (uint64_t)((x * tile_bytes) >> 4);
        const uint64_t kd = kdesc0 + (uint64_t)((st * 2 * tile_bytes) >> 4);
        for (int kk = 0; kk < d / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
          umma_bf16_ss(tmem + x * 256, qd + off, kd + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&ctl->s_full[x]);
      };
      // PV of tile x for its block j (stage st): waits for P (and, on a unit's
      // first block, for the epilogue to have read O)
      auto issue_pv = [&](int x, int j, int st) -> bool {
        // keys 0-63 as soon as their P is published, keys 64-127 after the rest
        if (!mbar_wait(&ctl->p_half[x], (uint32_t)(bt[x] & 1)) ||
            (j == 0 && !mbar_wait(&ctl->o_free[x], (ut[x] + 1) & 1)))
          return false;
        tc_fence_after();
        const uint64_t vd = vdesc0 + (uint64_t)((st * 2 * tile_bytes) >> 4);
        const uint32_t pcol = tmem + x * 256, ocol = pcol + 128;
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16_ts(ocol, pcol + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        if (!mbar_wait(&ctl->p_full[x], (uint32_t)(bt[x] & 1))) return false;
        tc_fence_after();
        for (int kk = 4; kk < 8; ++kk)
          umma_bf16_ts(ocol, pcol + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), idesc_o, 1u);
        umma_commit(&ctl->pv_done[x]);
        ++bt[x];
        return true;
      };
      while (ok && !*abort_flag) {
        const TileUnit* R = wait_unit(n);
        if (R == nullptr) { ok = false; break; }
        const int nblk = R->nblk, ntl = R->ntl;
        release_unit(n, false);
        if (nblk < 0) break;
        for (int j = 0; j < nblk && ok; ++j, ++kvc) {
          const int st = (int)(kvc & 1);
          if (!mbar_wait(&ctl->k_full[st], (uint32_t)((kvc >> 1) & 1)) ||
              !mbar_wait(&ctl->v_full[st], (uint32_t)((kvc >> 1) & 1)) ||
              (j == 0 && !mbar_wait(&ctl->q_full[0], ut[0] & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s(0, st);
          if (j == nblk - 1) umma_commit(&ctl->q_empty[0]);
          if (ntl == 2) {
            if (j > 0) {
              // tile 1's PV of the previous block; then both tiles are done with it
              if (!issue_pv(1, j - 1, st ^ 1)) { ok = false; break; }
              umma_commit(&ctl->kv_empty[st ^ 1]);
            }
            if (j == 0 && !mbar_wait(&ctl->q_full[1], ut[1] & 1)) { ok = false; break; }
            tc_fence_after();
            issue_s(1, st);
            if (j == nblk - 1) umma_commit(&ctl->q_empty[1]);
          }
          if (!issue_pv(0, j, st)) { ok = false; break; }
          if (ntl == 1) umma_commit(&ctl->kv_empty[st]);
        }
        if (ok && ntl == 2 && nblk > 0) {
          const int st = (int)((kvc - 1) & 1);
          if (!issue_pv(1, nblk - 1, st)) ok = false;
          else umma_commit(&ctl->kv_empty[st]);
        }
#pragma unroll
        for (int x = 0; x < 2; ++x)
          if (x < ntl) ++ut[x];
        ++n;
      }
      if (!ok) {
        report_error(p.err, MSA_ERR_TIMEOUT, kSiteTileMma, n, 0);
        *abort_flag = 1;
      }
      umma_commit(&ctl->mma_done[0]);
      mbar_wait(&ctl->mma_done[0], 0);
    }
  } else if (warp >= 4 && warp < 12) {
    // ----------------------------------------------------- online softmax
    const int x = (warp - 4) >> 2;            // MMA tile of this warpgroup
    const int wq = warp & 3;                  // TMEM lane quarter
    const int r = 32 * wq + lane;             // tile row
    const uint32_t lane_off = static_cast<uint32_t>(32 * wq) << 16;
    const uint32_t s_col = tmem + x * 256 + lane_off;   // S, then P
    const uint32_t o_col = s_col + 128;
    const int ql = r / RQ, hi = r - ql * RQ;
    const float sl2 = p.scale_log2;
    int n = 0, ut = 0;
    int64_t bt = 0;
    while (!*abort_flag) {
      const TileUnit* R = wait_unit(n);
      if (R == nullptr) break;
      const int nblk = R->nblk;
      if (nblk < 0) { release_unit(n, true); break; }
      if (x >= R->ntl) { release_unit(n, true); ++n; continue; }
      const int qi = x * qpt + ql;
      const bool valid = ql < qpt && qi < R->nq && hi < Hg;
      const int64_t t = R->r0 + qi;
      const int64_t pos = valid ? (int64_t)R->Sb - R->Tb + (t - R->qrow0) : -1;
      const int bk = kMode == kModeDense ? kBk : p.bk;
      const int lb = valid ? (int)(pos / bk) : -1;
      uint64_t mem = 0;
      if (kMode == kModeTiles && valid) mem = p.dmember[(t - p.t0) * G + R->g];
      float m_run = -INFINITY, l_run = 0.f;
      bool failed = false;
      for (int j = 0; j < nblk; ++j, ++bt) {
        const int blk = kMode == kModeDense ? j : R->blk[j];
        const bool member = valid && (kMode != kModeTiles || ((mem >> j) & 1ull)) && blk <= lb;
        int limit = -1;                          // last attended key of the block, -1: none
        if (member) limit = blk < lb ? bk - 1 : (int)(pos - (int64_t)blk * bk);
        if (!mbar_wait(&ctl->s_full[x], (uint32_t)(bt & 1))) {
          report_error(p.err, MSA_ERR_TIMEOUT, kSiteTileSoftmax, (int)bt, 0);
          failed = true;
          break;
        }
        tc_fence_after();
        uint32_t rr[32];
        float mx = -INFINITY;
        const bool all_full = __all_sync(0xffffffffu, limit == kBk - 1);
        const bool any_row = __any_sync(0xffffffffu, limit >= 0);
        if (all_full) {
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            tmem_ld32(s_col + 32 * c4, rr);
            tmem_ld_wait();
            float mm[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) mm[q] = fmaxf(__uint_as_float(rr[2 * q]), __uint_as_float(rr[2 * q + 1]));
#pragma unroll
            for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
              for (int q = 0; q < w; ++q) mm[q] = fmaxf(mm[q], mm[q + w]);
            mx = fmaxf(mx, mm[0]);
          }
        } else if (any_row) {
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            tmem_ld32(s_col + 32 * c4, rr);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q)
              mx = fmaxf(mx, 32 * c4 + q <= limit ? __uint_as_float(rr[q]) : -INFINITY);
          }
        }
        const float mb = limit >= 0 ? mx * sl2 : -INFINITY;
        float m_new = m_run, alpha = 1.f;
        if (mb > m_run) {
          if (m_run == -INFINITY) {
            m_new = mb;                          // first keys of this row: O row is still zero
          } else if (mb > m_run + kRescaleLog2) {
            m_new = mb;
            alpha = exp2f(m_run - mb);
          }
        }
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          // rescale this warp's O rows once the previous PV of this tile has landed
          // (before any of this block's P is published: PV(j) accumulates into O)
          if (!mbar_wait(&ctl->pv_done[x], (uint32_t)((bt + 1) & 1))) {
            report_error(p.err, MSA_ERR_TIMEOUT, kSiteTileSoftmax, (int)bt, 1);
            failed = true;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < d / 32; ++c) {
            tmem_ld32(o_col + 32 * c, rr);
            tmem_ld_wait();
            uint32_t lo[16], up[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              lo[q] = __float_as_uint(__uint_as_float(rr[q]) * alpha);
              up[q] = __float_as_uint(__uint_as_float(rr[16 + q]) * alpha);
            }
            tmem_st16(o_col + 32 * c, lo);
            tmem_st16(o_col + 32 * c + 16, up);
          }
        }
        // P of keys 0-63 is published first, so that the PV MMA can start on it
        auto publish_half = [&]() {
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->p_half[x]);
        };
        float lsum = 0.f;
        if (!any_row) {
          uint32_t z[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) z[q] = 0u;
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            tmem_st16(s_col + 16 * c4, z);
            if (c4 == 1) publish_half();
          }
        } else if (all_full) {
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            tmem_ld32(s_col + 32 * c4, rr);
            tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const float p0 = ex2_approx(fmaf(__uint_as_float(rr[2 * q]), sl2, -m_new));
              const float p1 = ex2_approx(fmaf(__uint_as_float(rr[2 * q + 1]), sl2, -m_new));
              lsum += p0 + p1;
              pk[q] = pack_bf16x2(p0, p1);
            }
            tmem_st16(s_col + 16 * c4, pk);
            if (c4 == 1) publish_half();
          }
        } else {
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            tmem_ld32(s_col + 32 * c4, rr);
            tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const int c0 = 32 * c4 + 2 * q;
              const float x0 = fmaf(__uint_as_float(rr[2 * q]), sl2, -m_new);
              const float x1 = fmaf(__uint_as_float(rr[2 * q + 1]), sl2, -m_new);
              const float p0 = ex2_approx(c0 <= limit ? x0 : -INFINITY);
              const float p1 = ex2_approx(c0 + 1 <= limit ? x1 : -INFINITY);
              lsum += p0 + p1;
              pk[q] = pack_bf16x2(p0, p1);
            }
            tmem_st16(s_col + 16 * c4, pk);
            if (c4 == 1) publish_half();
          }
        }
        l_run = l_run * alpha + lsum;
        m_run = m_new;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->p_full[x]);
      }
      if (failed) { *abort_flag = 1; break; }
      // final row statistics for the epilogue, once it has read the previous unit's
      if (!mbar_wait(&ctl->o_free[x], (ut + 1) & 1)) {
        report_error(p.err, MSA_ERR_TIMEOUT, kSiteTileSoftmax, ut, 2);
        *abort_flag = 1;
        break;
      }
      ctl->row_m[x][r] = m_run;
      ctl->row_l[x][r] = l_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->stats_full[x]);
      ++ut;
      release_unit(n, true);
      ++n;
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ epilogue
    const int wq = warp & 3;
    const int r = 32 * wq + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * wq) << 16;
    const int ql = r / RQ, hi = r - ql * RQ;
    int n = 0, ut[2] = {0, 0};
    int64_t bt[2] = {0, 0};
    bool failed = false;
    while (!*abort_flag && !failed) {
      const TileUnit* R = wait_unit(n);
      if (R == nullptr) break;
      const int nblk = R->nblk;
      if (nblk < 0) { release_unit(n, true); break; }
      const int g = R->g, ntl = R->ntl;
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        if (x >= ntl || failed) continue;
        const int qi = x * qpt + ql;
        const bool valid = ql < qpt && qi < R->nq && hi < Hg;
        const int64_t t = R->r0 + qi;
        if (!mbar_wait(&ctl->stats_full[x], ut[x] & 1) ||
            !mbar_wait(&ctl->pv_done[x], (uint32_t)((bt[x] + nblk - 1) & 1))) {
          report_error(p.err, MSA_ERR_TIMEOUT, kSiteTileSoftmax, ut[x], 3);
          failed = true;
          continue;
        }
        tc_fence_after();
        const float l = ctl->row_l[x][r], m = ctl->row_m[x][r];
        int32_t state = kDenseComplete;
        if (kMode == kModeTiles && valid) state = p.dstate[(t - p.t0) * G + g];
        const bool has = valid && l > 0.f && state >= 0;
        const bool complete = (state & kDenseComplete) != 0;
        const float inv_l = has ? 1.f / l : 0.f;
        const float lse_v = (m + __log2f(l)) * 0.69314718055994530942f;
        const int h = g * Hg + hi;
        const uint32_t o_col = tmem + x * 256 + 128 + lane_off;
        int64_t unit = 0;
        if (has && !complete) unit = ((t - p.t0) * G + g) * p.k;   // packed position 0
        uint32_t rr[32];
#pragma unroll 1
        for (int c4 = 0; c4 < d / 32; ++c4) {
          tmem_ld32(o_col + 32 * c4, rr);
          tmem_ld_wait();
          if (has) {
            if (complete) {
              uint4* dst = reinterpret_cast<uint4*>(p.out + (t * H + h) * d + 32 * c4);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(rr[8 * q + 0]) * inv_l, __uint_as_float(rr[8 * q + 1]) * inv_l);
                w.y = pack_bf16x2(__uint_as_float(rr[8 * q + 2]) * inv_l, __uint_as_float(rr[8 * q + 3]) * inv_l);
                w.z = pack_bf16x2(__uint_as_float(rr[8 * q + 4]) * inv_l, __uint_as_float(rr[8 * q + 5]) * inv_l);
                w.w = pack_bf16x2(__uint_as_float(rr[8 * q + 6]) * inv_l, __uint_as_float(rr[8 * q + 7]) * inv_l);
                __stcs(dst + q, w);            // write-once: evict-first in L2
              }
            } else {
              // partial layout per unit: [d/8 chunks][Hg heads][8 values]
              __half* dst = p.part_acc + unit * Hg * d + hi * 8;
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                uint4 w;
                w.x = pack_f16x2(__uint_as_float(rr[8 * q + 0]) * inv_l, __uint_as_float(rr[8 * q + 1]) * inv_l);
                w.y = pack_f16x2(__uint_as_float(rr[8 * q + 2]) * inv_l, __uint_as_float(rr[8 * q + 3]) * inv_l);
                w.z = pack_f16x2(__uint_as_float(rr[8 * q + 4]) * inv_l, __uint_as_float(rr[8 * q + 5]) * inv_l);
                w.w = pack_f16x2(__uint_as_float(rr[8 * q + 6]) * inv_l, __uint_as_float(rr[8 * q + 7]) * inv_l);
                __stcs(reinterpret_cast<uint4*>(dst + (4 * c4 + q) * Hg * 8), w);
              }
            }
          }
        }
        if (has) {
          if (complete) {
            if (p.lse != nullptr) __stcs(p.lse + t * H + h, lse_v);
          } else {
            __stcs(p.part_lse + unit * Hg + hi, lse_v);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->o_free[x]);
        ++ut[x];
        bt[x] += nblk;
      }
      if (failed) { *abort_flag = 1; break; }
      release_unit(n, true);
      ++n;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int make_tile_maps(CUtensorMap* tm_k, CUtensorMap* tm_v, CUtensorMap* tm_q, const void* q, const void* key,
                   const void* value, int64_t total_q, int64_t total_k, int H, int G, int d) {
  {
    const uint64_t dims[3] = {(uint64_t)d, (uint64_t)G, (uint64_t)total_k};
    const uint64_t strides[2] = {(uint64_t)d * 2, (uint64_t)G * d * 2};
    const uint32_t box[3] = {64u, 1u, 128u};
    int rc = make_tmap_bf16(tm_k, key, 3, dims, strides, box, 128);
    if (rc) return rc;
    rc = make_tmap_bf16(tm_v, value, 3, dims, strides, box, 128);
    if (rc) return rc;
  }
  const int hg = H / G;
  const int RQ = hg < 8 ? 8 : hg;
  const uint64_t dims[3] = {(uint64_t)d, (uint64_t)H, (uint64_t)total_q};
  const uint64_t strides[2] = {(uint64_t)d * 2, (uint64_t)H * d * 2};
  const uint32_t box[3] = {64u, (uint32_t)RQ, (uint32_t)(128 / RQ)};
  return make_tmap_bf16(tm_q, q, 3, dims, strides, box, 128);
}

template <int kMode>
int launch_tile_attn_kernel(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_q,
                            const TileParams& prm, cudaStream_t st) {
  const size_t smem = 1024 + 6 * (size_t)128 * prm.d * 2 + sizeof(TileCtl);
  static_assert(1024 + 6 * 128 * 128 * 2 + sizeof(TileCtl) <= 227 * 1024, "shared memory budget (d = 128)");
  cudaError_t e =
      cudaFuncSetAttribute(tile_attn_kernel<kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  tile_attn_kernel<kMode><<<nsm, kTileThreads, smem, st>>>(tm_k, tm_v, tm_q, prm);
  return (int)cudaGetLastError();
}

}  // namespace

int tile_queries(int H, int G) {
  const int hg = H / G;
  return 2 * (128 / (hg < 8 ? 8 : hg));
}

int tile_default_theta(int UQ) { return (5 * UQ + 7) / 8; }   // ceil(5/8 x tile queries), by measurement

int launch_tile_plan(const AttnArgs& a, int theta, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int UQ = tile_queries(a.H, a.G);
  const int64_t nunits = (a.t1 - a.t0 + UQ - 1) / UQ;
  const int64_t nwarps = nunits * a.G;
  if (nwarps <= 0) return 0;
  ProfScope ps("tile_plan", stream);
  tile_plan_kernel<<<(unsigned)((nwarps + kPlanWarps - 1) / kPlanWarps), kPlanWarps * 32, 0, st>>>(
      a.sel, a.t0, a.t1, a.G, a.k, UQ, theta, a.batch, a.cu_q, a.unit_blk, a.unit_nblk, a.unit_list, a.dmask,
      a.dstate, a.dmember, a.clist, a.tile_ctr);
  return (int)cudaGetLastError();
}

int launch_tile_attn(const AttnArgs& a, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  alignas(64) CUtensorMap tm_k, tm_v, tm_q;
  int rc = make_tile_maps(&tm_k, &tm_v, &tm_q, a.q, a.key, a.value, a.total_q, a.total_k, a.H, a.G, a.d);
  if (rc) return rc;
  TileParams prm{};
  prm.unit_list = a.unit_list; prm.unit_blk = a.unit_blk; prm.unit_nblk = a.unit_nblk;
  prm.dmember = a.dmember; prm.dstate = a.dstate;
  prm.nunits = a.tile_ctr + 1; prm.ticket = a.tile_ctr + 2;
  prm.cu_q = a.cu_q; prm.cu_k = a.cu_k;
  prm.batch = a.batch; prm.H = a.H; prm.G = a.G; prm.d = a.d; prm.k = a.k; prm.UQ = tile_queries(a.H, a.G);
  prm.bk = a.B_k;
  prm.scale_log2 = a.sm_scale * 1.4426950408889634f;
  prm.t0 = a.t0; prm.t1 = a.t1;
  prm.out = reinterpret_cast<__nv_bfloat16*>(a.out);
  prm.lse = a.lse;
  prm.part_acc = reinterpret_cast<__half*>(a.part_acc);
  prm.part_lse = a.part_lse;
  prm.err = a.err;
  ProfScope ps("tile_attn", stream);
  return launch_tile_attn_kernel<kModeTiles>(tm_k, tm_v, tm_q, prm, st);
}

int launch_rows_attn(const AttnArgs& a, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t rows = a.t1 - a.t0;
  if (rows <= 0) return 0;
  cudaError_t e = cudaMemsetAsync(a.tile_ctr, 0, sizeof(int32_t) * 4, st);
  if (e != cudaSuccess) return (int)e;
  alignas(64) CUtensorMap tm_k, tm_v, tm_q;
  const int64_t krows = a.block_table != nullptr ? a.num_pages * kBk : a.total_k;
  int rc = make_tile_maps(&tm_k, &tm_v, &tm_q, a.q, a.key, a.value, a.total_q, krows, a.H, a.G, a.d);
  if (rc) return rc;
  TileParams prm{};
  prm.nunits = nullptr; prm.nunits_host = rows * a.G; prm.ticket = a.tile_ctr + 2;
  prm.sel = a.sel;
  prm.block_table = a.block_table; prm.max_blocks = a.max_blocks; prm.num_pages = a.num_pages;
  prm.cu_q = a.cu_q; prm.cu_k = a.cu_k;
  prm.batch = a.batch; prm.H = a.H; prm.G = a.G; prm.d = a.d; prm.k = a.k; prm.UQ = 1;
  prm.bk = a.B_k;
  prm.scale_log2 = a.sm_scale * 1.4426950408889634f;
  prm.t0 = a.t0; prm.t1 = a.t1;
  prm.out = reinterpret_cast<__nv_bfloat16*>(a.out);
  prm.lse = a.lse;
  prm.err = a.err;
  ProfScope ps("rows_attn", stream);
  return launch_tile_attn_kernel<kModeRows>(tm_k, tm_v, tm_q, prm, st);
}

size_t dense_scratch_bytes(int32_t batch) { return align_up(sizeof(int32_t) * (batch + 1), 256) + 256; }

int launch_dense_attn(const DenseArgs& a, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t* seq_units = reinterpret_cast<int32_t*>(a.scratch);
  int32_t* ctr = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(a.scratch) +
                                            align_up(sizeof(int32_t) * (a.batch + 1), 256));
  const int UQ = tile_queries(a.H, a.G);
  {
    ProfScope ps("dense_units", stream);
    dense_units_kernel<<<1, 32, 0, st>>>(a.cu_q, a.batch, UQ, a.G, seq_units, ctr);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  alignas(64) CUtensorMap tm_k, tm_v, tm_q;
  int rc = make_tile_maps(&tm_k, &tm_v, &tm_q, a.q, a.key, a.value, a.total_q, a.total_k, a.H, a.G, a.d);
  if (rc) return rc;
  TileParams prm{};
  prm.seq_units = seq_units;
  prm.nunits = ctr + 1; prm.ticket = ctr + 2;
  prm.cu_q = a.cu_q; prm.cu_k = a.cu_k;
  prm.batch = a.batch; prm.H = a.H; prm.G = a.G; prm.d = a.d; prm.k = 1; prm.UQ = UQ;
  prm.bk = kBk;
  prm.scale_log2 = a.sm_scale * 1.4426950408889634f;
  prm.t0 = 0; prm.t1 = a.total_q;
  prm.out = reinterpret_cast<__nv_bfloat16*>(a.out);
  prm.lse = a.lse;
  prm.err = a.err;
  ProfScope ps("dense_attn", stream);
  return launch_tile_attn_kernel<kModeDense>(tm_k, tm_v, tm_q, prm, st);
}

}  // namespace msa
