// C ABI of libmsa (declared in include/msa.h): argument checks, workspace
// layout, tensor-map creation and the launch sequence of each entry point.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <mutex>

#include "msa_internal.h"
#include "msa_kl.h"
#include "msa_window.h"
#include "msa_bwd.h"
#include "msa_policy.h"
#include "msa_gather.h"

using namespace msa;

namespace msa {

static bool shape_ok(const msa_shape_t* s) {
  return s != nullptr && s->H > 0 && s->G > 0 && s->d > 0 && s->d_idx > 0 && s->B_k > 0 && s->k > 0;
}

msa_status_t check_shape(const msa_shape_t* s) {
  if (!shape_ok(s)) return MSA_ERR_INVALID_ARG;
  if (s->H % s->G != 0) return MSA_ERR_INVALID_ARG;
  const int hg = s->H / s->G;
  if (hg != 4 && hg != 8 && hg != 16) return MSA_ERR_UNSUPPORTED;
  if (s->G != 1 && s->G != 2 && s->G != 4) return MSA_ERR_UNSUPPORTED;
  if (s->d != 64 && s->d != 128) return MSA_ERR_UNSUPPORTED;
  if (s->d_idx != 32 && s->d_idx != 64 && s->d_idx != 128) return MSA_ERR_UNSUPPORTED;
  if (s->B_k != 32 && s->B_k != 64 && s->B_k != kBk) return MSA_ERR_UNSUPPORTED;
  if (s->k < 1 || s->k > kMaxK) return MSA_ERR_UNSUPPORTED;
  if (!(s->sm_scale > 0.f) || s->sm_scale != s->sm_scale) return MSA_ERR_INVALID_ARG;
  return MSA_OK;
}

msa_status_t check_seqs(const msa_varlen_t* v) {
  if (v == nullptr || v->cu_q == nullptr || v->cu_k == nullptr) return MSA_ERR_INVALID_ARG;
  if (v->batch < 1 || v->total_q < 0 || v->total_k < 1 || v->max_q_len < 0 || v->max_k_len < 1)
    return MSA_ERR_INVALID_ARG;
  if (v->total_q > v->total_k || v->max_q_len > v->max_k_len) return MSA_ERR_INVALID_ARG;
  if (v->max_q_len > v->total_q || v->max_k_len > v->total_k) return MSA_ERR_INVALID_ARG;  // a length beyond its total
  if (v->total_k > (int64_t)INT32_MAX - 256 || v->total_q > (int64_t)INT32_MAX / kMaxK) return MSA_ERR_UNSUPPORTED;
  return MSA_OK;
}

// Entry points built for 128-token blocks only (the training-side kernels,
// the selection variants and paged caches, whose pages are 128-row blocks).
msa_status_t check_shape_bk128(const msa_shape_t* s) {
  const msa_status_t st = check_shape(s);
  if (st != MSA_OK) return st;
  return s->B_k == kBk ? MSA_OK : MSA_ERR_UNSUPPORTED;
}

}  // namespace msa

namespace {

// Query-tile threshold (msa_set_tile_threshold): -1 automatic, 0 off.
std::atomic<int> g_tile_theta{-1};
// Query rows per planning window of the KV-outer lists (msa_set_attn_window).
std::atomic<int> g_attn_window{kDefaultWindow};
// SMs that msa_prefill gives a pass's combine while the next pass's index
// top-k runs on the others (msa_set_prefill_overlap; 0: no overlap, the
// default: on B200 a combine on a slice of the SMs is latency-bound and
// outlasts the index pass it would hide behind).
constexpr int kDefaultOverlapSms = 0;
std::atomic<int> g_overlap_sms{kDefaultOverlapSms};

// Per device: the second stream of msa_prefill and its two events, created on
// first use and kept for the life of the process.  The mutex is held while a
// call enqueues its work, so concurrent calls never interleave their records
// and waits on the shared events.
constexpr int kMaxSideDevices = 64;
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t main_done = nullptr;   // a pass's main phase is done (its partials are written)
  cudaEvent_t comb_done = nullptr;   // a pass's combine is done (its workspace may be reused)
};
std::mutex g_side_mu;
SideStream g_side[kMaxSideDevices];

// Called with g_side_mu held.
SideStream* side_stream() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxSideDevices) return nullptr;
  SideStream& s = g_side[dev];
  if (s.stream == nullptr) {
    cudaStream_t st = nullptr;
    cudaEvent_t e0 = nullptr, e1 = nullptr;
    if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (cudaEventCreateWithFlags(&e0, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&e1, cudaEventDisableTiming) != cudaSuccess) {
      if (e0) cudaEventDestroy(e0);
      cudaStreamDestroy(st);
      return nullptr;
    }
    s.stream = st; s.main_done = e0; s.comb_done = e1;
  }
  return &s;
}

constexpr size_t kAlign = 256;

bool ws_ok(const void* ws, size_t have, size_t need) {
  return ws != nullptr && (reinterpret_cast<uintptr_t>(ws) % kAlign) == 0 && have >= need;
}

int64_t total_blocks_bound(const msa_varlen_t* v, int B_k) { return (v->total_k + B_k - 1) / B_k + v->batch; }

// Slices of a sparse-attention workspace for chunks of `rows` query rows.
struct AttnLayout {
  size_t blk_off, counts, cursor, tile_sums, nitems, entries, items, part_acc, part_lse;
  size_t unit_blk, unit_nblk, unit_list, dmask, dstate, dmember, clist, tile_ctr, total;
  int64_t nlists, max_items;
  int32_t qpi, win;
};

AttnLayout attn_layout(const msa_shape_t* s, const msa_varlen_t* v, int64_t rows) {
  AttnLayout L{};
  const int hg = s->H / s->G;
  const int qpt = 128 / (hg < 8 ? 8 : hg);            // queries per 128-row tile
  L.qpi = 8 * qpt < kMaxItemQueries ? 8 * qpt : kMaxItemQueries;
  L.nlists = (int64_t)s->G * total_blocks_bound(v, s->B_k);
  L.win = attn_window_rows();
  const int64_t nkeys = ((rows + L.win - 1) / L.win) * L.nlists;
  const int64_t nentries = rows * s->G * s->k;
  L.max_items = nentries / L.qpi + (nkeys < nentries ? nkeys : nentries) + 1;
  size_t off = kWsHeader;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, kAlign);
    return o;
  };
  L.blk_off = take(sizeof(int32_t) * (v->batch + 1));
  L.counts = take(sizeof(int32_t) * nkeys);
  L.cursor = take(sizeof(int32_t) * nkeys);
  L.tile_sums = take(sizeof(int32_t) * 2 * ((nkeys + kScanTile - 1) / kScanTile + 1));
  L.nitems = take(sizeof(int32_t) * 4);
  L.entries = take(sizeof(uint32_t) * nentries);
  L.items = take(sizeof(Item) * L.max_items);
  L.part_acc = take((size_t)nentries * hg * s->d * 2);
  L.part_lse = take((size_t)nentries * hg * 4);
  const int UQ = tile_queries(s->H, s->G);
  const int64_t nunits = ((rows + UQ - 1) / UQ) * s->G;
  L.unit_blk = take(sizeof(int32_t) * nunits * kMaxDense);
  L.unit_nblk = take(sizeof(int32_t) * nunits);
  L.unit_list = take(sizeof(int32_t) * nunits);
  L.dmask = take(sizeof(uint32_t) * rows * s->G);
  L.dstate = take(sizeof(int32_t) * rows * s->G);
  L.dmember = take(sizeof(uint64_t) * rows * s->G);
  L.clist = take(sizeof(uint2) * rows * s->G);
  L.tile_ctr = take(sizeof(int32_t) * 4);
  L.total = off;
  return L;
}

// Threshold for this call: the query tiles need several queries per sequence.
int tile_theta(const msa_shape_t* s, const msa_varlen_t* v) {
  const int set = g_tile_theta.load(std::memory_order_relaxed);
  if (set == 0 || v->max_q_len <= 1) return 0;
  return set < 0 ? tile_default_theta(tile_queries(s->H, s->G)) : set;
}

int64_t chunk_rows(const msa_varlen_t* v, int64_t q_chunk) {
  if (q_chunk <= 0 || q_chunk > v->total_q) return v->total_q;
  return q_chunk;
}

// Attention arguments of a call whose workspace `base` has layout L.
AttnArgs attn_args(const msa_shape_t* shape, const msa_varlen_t* seqs, const AttnLayout& L, uint8_t* base,
                   const void* q, const void* k, const void* v, const int32_t* sel, void* out, float* lse) {
  AttnArgs a{};
  a.q = q; a.key = k; a.value = v; a.sel = sel; a.out = out; a.lse = lse;
  a.cu_q = seqs->cu_q; a.cu_k = seqs->cu_k;
  a.batch = seqs->batch; a.H = shape->H; a.G = shape->G; a.d = shape->d; a.k = shape->k;
  a.B_k = shape->B_k;
  a.sm_scale = shape->sm_scale;
  a.total_q = seqs->total_q; a.total_k = seqs->total_k;
  a.max_q_len = seqs->max_q_len; a.max_k_len = seqs->max_k_len;
  a.err = reinterpret_cast<DevError*>(base);
  a.blk_off = reinterpret_cast<int32_t*>(base + L.blk_off);
  a.counts = reinterpret_cast<int32_t*>(base + L.counts);
  a.cursor = reinterpret_cast<int32_t*>(base + L.cursor);
  a.tile_sums = reinterpret_cast<int32_t*>(base + L.tile_sums);
  a.nitems = reinterpret_cast<int32_t*>(base + L.nitems);
  a.entries = reinterpret_cast<uint32_t*>(base + L.entries);
  a.items = reinterpret_cast<Item*>(base + L.items);
  a.max_items = L.max_items;
  a.nlists = L.nlists;
  a.win_rows = L.win;
  a.part_acc = base + L.part_acc;
  a.part_lse = reinterpret_cast<float*>(base + L.part_lse);
  a.queries_per_item = L.qpi;
  a.theta = tile_theta(shape, seqs);
  a.unit_blk = reinterpret_cast<int32_t*>(base + L.unit_blk);
  a.unit_nblk = reinterpret_cast<int32_t*>(base + L.unit_nblk);
  a.unit_list = reinterpret_cast<int32_t*>(base + L.unit_list);
  a.dmask = reinterpret_cast<uint32_t*>(base + L.dmask);
  a.dstate = reinterpret_cast<int32_t*>(base + L.dstate);
  a.dmember = reinterpret_cast<uint64_t*>(base + L.dmember);
  a.clist = reinterpret_cast<uint2*>(base + L.clist);
  a.tile_ctr = reinterpret_cast<int32_t*>(base + L.tile_ctr);
  return a;
}

msa_status_t attn_common(const msa_shape_t* shape, const msa_varlen_t* seqs, const void* q, const void* k,
                         const void* v, const int32_t* sel, void* out, float* lse, int64_t q_chunk, void* ws,
                         size_t ws_bytes, void* stream) {
  msa_status_t st = check_shape(shape);
  if (st != MSA_OK) return st;
  st = check_seqs(seqs);
  if (st != MSA_OK) return st;
  // no queries: nothing is read or written (empty tensors may have no storage)
  if (seqs->total_q > 0 && (!q || !k || !v || !sel || !out)) return MSA_ERR_INVALID_ARG;
  const int64_t rows = chunk_rows(seqs, q_chunk);
  const AttnLayout L = attn_layout(shape, seqs, rows);
  if (!ws_ok(ws, ws_bytes, L.total)) return MSA_ERR_WORKSPACE;
  if (cudaMemsetAsync(ws, 0, sizeof(DevError), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (seqs->total_q == 0) return MSA_OK;
  AttnArgs a = attn_args(shape, seqs, L, static_cast<uint8_t*>(ws), q, k, v, sel, out, lse);
  for (int64_t t0 = 0; t0 < seqs->total_q; t0 += rows) {
    a.t0 = t0;
    a.t1 = t0 + rows < seqs->total_q ? t0 + rows : seqs->total_q;
    // one query per sequence: each (query, group) attends its selected blocks
    // query-major (no lists, partials or combine)
    const int rc = seqs->max_q_len <= 1 ? launch_rows_attn(a, stream) : launch_sparse_attn_pass(a, stream);
    if (rc != 0) return MSA_ERR_CUDA;
  }
  return MSA_OK;
}

// Paged decode: workspace slices and argument checks.
struct PagedLayout {
  size_t cu_q, cu_k, tile_ctr, idx_scratch, total;
  int64_t total_k;   // upper bound of the cached tokens
};

msa_status_t check_paged(const msa_shape_t* s, const msa_paged_t* pg) {
  msa_status_t st = check_shape_bk128(s);
  if (st != MSA_OK) return st;
  if (pg == nullptr || pg->seqlens == nullptr || pg->block_table == nullptr) return MSA_ERR_INVALID_ARG;
  if (pg->batch < 1 || pg->max_blocks < 1 || pg->num_pages < 1 || pg->max_seqlen < 1) return MSA_ERR_INVALID_ARG;
  if (pg->max_seqlen > (int64_t)pg->max_blocks * kBk) return MSA_ERR_INVALID_ARG;
  // key rows are int32 coordinates; cached tokens are summed in int32
  if (pg->num_pages > (INT32_MAX - kBk) / kBk) return MSA_ERR_UNSUPPORTED;
  if ((int64_t)pg->batch * pg->max_blocks * kBk > (int64_t)INT32_MAX - 256) return MSA_ERR_UNSUPPORTED;
  return MSA_OK;
}

PagedLayout paged_layout(const msa_shape_t* s, const msa_paged_t* pg) {
  PagedLayout L{};
  L.total_k = (int64_t)pg->batch * pg->max_blocks * kBk;
  size_t off = kWsHeader;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, kAlign);
    return o;
  };
  L.cu_q = take(sizeof(int32_t) * (pg->batch + 1));
  L.cu_k = take(sizeof(int32_t) * (pg->batch + 1));
  L.tile_ctr = take(sizeof(int32_t) * 4);
  L.idx_scratch = take(decode_index_scratch_bytes(pg->batch, L.total_k, s->G, kBk));
  L.total = off;
  return L;
}

}  // namespace

namespace msa {

int attn_window_rows() { return g_attn_window.load(std::memory_order_relaxed); }

int make_tmap_bf16(void* tmap_out, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                   const uint32_t* box, int swizzle_bytes) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (encode == nullptr) return (int)cudaErrorNotSupported;
  cuuint64_t gdim[5];
  cuuint64_t gstr[4];
  cuuint32_t bdim[5], estr[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estr[i] = 1;
    if (i + 1 < rank) gstr[i] = strides_bytes[i];
  }
  const CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE;
  const CUresult r = encode(reinterpret_cast<CUtensorMap*>(tmap_out), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                            (cuuint32_t)rank, const_cast<void*>(base), gdim, gstr, bdim, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : (int)cudaErrorInvalidValue;
}

}  // namespace msa

extern "C" {

const char* msa_version(void) { return "msa-b200 0.1 (sm_100a)"; }

size_t msa_index_topk_workspace_size(const msa_shape_t* shape, const msa_varlen_t* seqs) {
  if (check_shape(shape) != MSA_OK || check_seqs(seqs) != MSA_OK) return 0;
  if (seqs->max_q_len > 1 && seqs->batch > kMaxBatchTiles) return 0;
  size_t need = kWsHeader;
  if (seqs->max_q_len <= 1)
    need += align_up(decode_index_scratch_bytes(seqs->batch, seqs->total_k, shape->G, shape->B_k), kAlign);
  return need;
}

msa_status_t msa_index_topk(const msa_shape_t* shape, const msa_varlen_t* seqs, const void* q_idx,
                            const void* k_idx, int32_t* sel, void* ws, size_t ws_bytes, void* stream) {
  msa_status_t st = check_shape(shape);
  if (st != MSA_OK) return st;
  st = check_seqs(seqs);
  if (st != MSA_OK) return st;
  // prefill-shaped calls keep a per-sequence tile prefix in shared memory
  if (seqs->max_q_len > 1 && seqs->batch > kMaxBatchTiles) return MSA_ERR_UNSUPPORTED;
  if (seqs->total_q > 0 && (!q_idx || !k_idx || !sel)) return MSA_ERR_INVALID_ARG;
  const size_t need = msa_index_topk_workspace_size(shape, seqs);
  if (!ws_ok(ws, ws_bytes, need)) return MSA_ERR_WORKSPACE;
  if (cudaMemsetAsync(ws, 0, sizeof(DevError), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (seqs->total_q == 0) return MSA_OK;
  IndexTopkArgs a{};
  a.q_idx = q_idx; a.k_idx = k_idx; a.sel = sel;
  a.cu_q = seqs->cu_q; a.cu_k = seqs->cu_k;
  a.batch = seqs->batch; a.G = shape->G; a.d_idx = shape->d_idx; a.k = shape->k; a.B_k = shape->B_k;
  a.total_q = seqs->total_q; a.total_k = seqs->total_k;
  a.max_q_len = seqs->max_q_len; a.max_k_len = seqs->max_k_len;
  a.err = static_cast<DevError*>(ws);
  a.scratch = static_cast<uint8_t*>(ws) + kWsHeader;
  a.scratch_bytes = ws_bytes - kWsHeader;
  int rc;
  if (seqs->max_q_len <= 1) {
    rc = launch_index_topk_decode(a, stream);
  } else {
    rc = launch_index_topk_prefill(a, stream);
  }
  return rc == 0 ? MSA_OK : MSA_ERR_CUDA;
}

msa_status_t msa_index_topk_decode_candidates(const msa_shape_t* shape, const msa_varlen_t* seqs,
                                              const void* q_idx, const void* k_idx, int32_t all_blocks,
                                              int32_t* cand_ids, float* cand_scores, void* ws, size_t ws_bytes,
                                              void* stream) {
  msa_status_t st = check_shape(shape);
  if (st != MSA_OK) return st;
  st = check_seqs(seqs);
  if (st != MSA_OK) return st;
  if (seqs->max_q_len > 1) return MSA_ERR_INVALID_ARG;          // one query per sequence
  if (all_blocks != 0 && all_blocks != 1) return MSA_ERR_INVALID_ARG;
  const bool any = seqs->total_q > 0 && shape->k > 1;          // k = 1: no candidates, only the local block
  if (any && (!q_idx || !k_idx || !cand_ids || !cand_scores)) return MSA_ERR_INVALID_ARG;
  const size_t need = msa_index_topk_workspace_size(shape, seqs);
  if (!ws_ok(ws, ws_bytes, need)) return MSA_ERR_WORKSPACE;
  if (cudaMemsetAsync(ws, 0, sizeof(DevError), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (!any) return MSA_OK;
  IndexTopkArgs a{};
  a.q_idx = q_idx; a.k_idx = k_idx; a.sel = cand_ids; a.cand_score = cand_scores;
  a.all_blocks = all_blocks;
  a.cu_q = seqs->cu_q; a.cu_k = seqs->cu_k;
  a.batch = seqs->batch; a.G = shape->G; a.d_idx = shape->d_idx; a.k = shape->k; a.B_k = shape->B_k;
  a.total_q = seqs->total_q; a.total_k = seqs->total_k;
  a.max_q_len = seqs->max_q_len; a.max_k_len = seqs->max_k_len;
  a.err = static_cast<DevError*>(ws);
  a.scratch = static_cast<uint8_t*>(ws) + kWsHeader;
  a.scratch_bytes = ws_bytes - kWsHeader;
  return launch_index_topk_decode(a, stream) == 0 ? MSA_OK : MSA_ERR_CUDA;
}

size_t msa_sparse_attn_workspace_size(const msa_shape_t* shape, const msa_varlen_t* seqs, int64_t q_chunk) {
  if (check_shape(shape) != MSA_OK || check_seqs(seqs) != MSA_OK) return 0;
  return attn_layout(shape, seqs, chunk_rows(seqs, q_chunk)).total;
}

msa_status_t msa_sparse_attn_prefill(const msa_shape_t* shape, const msa_varlen_t* seqs, const void* q,
                                     const void* k, const void* v, const int32_t* sel, void* out, float* lse,
                                     int64_t q_chunk, void* ws, size_t ws_bytes, void* stream) {
  return attn_common(shape, seqs, q, k, v, sel, out, lse, q_chunk, ws, ws_bytes, stream);
}

size_t msa_prefill_workspace_size(const msa_shape_t* shape, const msa_varlen_t* seqs, int64_t q_chunk) {
  if (check_shape(shape) != MSA_OK || check_seqs(seqs) != MSA_OK) return 0;
  if (seqs->max_q_len <= 1 || seqs->batch > kMaxBatchTiles) return 0;
  return attn_layout(shape, seqs, chunk_rows(seqs, q_chunk)).total;
}

msa_status_t msa_prefill(const msa_shape_t* shape, const msa_varlen_t* seqs, const void* q, const void* k,
                         const void* v, const void* q_idx, const void* k_idx, int32_t* sel, void* out, float* lse,
                         int64_t q_chunk, void* ws, size_t ws_bytes, void* stream) {
  msa_status_t st = check_shape(shape);
  if (st != MSA_OK) return st;
  st = check_seqs(seqs);
  if (st != MSA_OK) return st;
  if (seqs->max_q_len <= 1) return MSA_ERR_INVALID_ARG;            // decode shapes: the decode calls
  if (seqs->batch > kMaxBatchTiles) return MSA_ERR_UNSUPPORTED;
  if (seqs->total_q > 0 && (!q || !k || !v || !q_idx || !k_idx || !sel || !out)) return MSA_ERR_INVALID_ARG;
  const int64_t rows = chunk_rows(seqs, q_chunk);
  const AttnLayout L = attn_layout(shape, seqs, rows);
  if (!ws_ok(ws, ws_bytes, L.total)) return MSA_ERR_WORKSPACE;
  cudaStream_t main = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(DevError), main) != cudaSuccess) return MSA_ERR_CUDA;
  if (seqs->total_q == 0) return MSA_OK;
  AttnArgs a = attn_args(shape, seqs, L, static_cast<uint8_t*>(ws), q, k, v, sel, out, lse);
  IndexTopkArgs ia{};
  ia.q_idx = q_idx; ia.k_idx = k_idx; ia.sel = sel;
  ia.cu_q = seqs->cu_q; ia.cu_k = seqs->cu_k;
  ia.batch = seqs->batch; ia.G = shape->G; ia.d_idx = shape->d_idx; ia.k = shape->k; ia.B_k = shape->B_k;
  ia.total_q = seqs->total_q; ia.total_k = seqs->total_k;
  ia.max_q_len = seqs->max_q_len; ia.max_k_len = seqs->max_k_len;
  ia.err = a.err;
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MSA_ERR_CUDA;
  const int64_t npass = (seqs->total_q + rows - 1) / rows;
  int csms = g_overlap_sms.load(std::memory_order_relaxed);
  if (csms > nsm / 2) csms = nsm / 2;
  std::unique_lock<std::mutex> lk(g_side_mu, std::defer_lock);
  SideStream* side = nullptr;
  if (npass > 1 && csms > 0) {
    lk.lock();
    side = side_stream();
    if (side == nullptr) return MSA_ERR_CUDA;
  }
  // Per pass p: index top-k of its rows (the tiles whose first row is in the
  // pass), the main phase, then the combine.  With a side stream, the combine
  // of pass p runs there on csms SMs while the index top-k of pass p + 1 runs
  // on the other SMs; the main phase of pass p + 1 waits for that combine (it
  // reuses the pass workspace).  The last pass combines on the caller's stream.
  bool ok = true;
  for (int64_t p = 0; p < npass && ok; ++p) {
    a.t0 = p * rows;
    a.t1 = a.t0 + rows < seqs->total_q ? a.t0 + rows : seqs->total_q;
    ia.row0 = a.t0;
    ia.row1 = p == npass - 1 ? seqs->total_q : a.t1;
    ia.grid = (side != nullptr && p > 0) ? nsm - csms : 0;
    ok = launch_index_topk_prefill(ia, stream) == 0;
    if (ok && side != nullptr && p > 0) ok = cudaStreamWaitEvent(main, side->comb_done, 0) == cudaSuccess;
    if (ok) ok = launch_sparse_attn_main(a, stream) == 0;
    if (!ok) break;
    if (side != nullptr && p < npass - 1) {
      ok = cudaEventRecord(side->main_done, main) == cudaSuccess &&
           cudaStreamWaitEvent(side->stream, side->main_done, 0) == cudaSuccess &&
           launch_sparse_attn_combine(a, side->stream, csms) == 0 &&
           cudaEventRecord(side->comb_done, side->stream) == cudaSuccess;
    } else {
      ok = launch_sparse_attn_combine(a, stream, 0) == 0;
    }
  }
  if (!ok && side != nullptr) {
    // the caller's stream still waits for whatever reached the side stream
    cudaEventRecord(side->comb_done, side->stream);
    cudaStreamWaitEvent(main, side->comb_done, 0);
  }
  return ok ? MSA_OK : MSA_ERR_CUDA;
}

int32_t msa_set_prefill_overlap(int32_t sms) {
  return g_overlap_sms.exchange(sms < 0 ? kDefaultOverlapSms : sms);
}

msa_status_t msa_sparse_attn_decode(const msa_shape_t* shape, const msa_varlen_t* seqs, const void* q,
                                    const void* k_cache, const void* v_cache, const int32_t* sel, void* out,
                                    float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (seqs != nullptr && seqs->max_q_len > 1) return MSA_ERR_INVALID_ARG;
  return attn_common(shape, seqs, q, k_cache, v_cache, sel, out, lse, 0, ws, ws_bytes, stream);
}

msa_status_t msa_combine(const msa_shape_t* shape, int64_t T, const void* part_acc, const float* part_lse,
                         const int32_t* sel, void* out, float* lse, void* stream) {
  msa_status_t st = check_shape(shape);
  if (st != MSA_OK) return st;
  if (T < 0) return MSA_ERR_INVALID_ARG;
  if (T == 0) return MSA_OK;                 // nothing to merge (pointers may be NULL)
  if (!part_acc || !part_lse || !sel || !out) return MSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(part_acc) | reinterpret_cast<uintptr_t>(part_lse)) & 15u)
    return MSA_ERR_INVALID_ARG;   // streamed with 16-byte bulk copies
  return launch_combine(part_acc, part_lse, sel, out, lse, T, shape->H, shape->G, shape->d, shape->k, stream) == 0
             ? MSA_OK
             : MSA_ERR_CUDA;
}

size_t msa_dense_attn_workspace_size(const msa_shape_t* shape, const msa_varlen_t* seqs) {
  if (check_shape(shape) != MSA_OK || check_seqs(seqs) != MSA_OK) return 0;
  return kWsHeader + dense_scratch_bytes(seqs->batch);
}

msa_status_t msa_dense_attn(const msa_shape_t* shape, const msa_varlen_t* seqs, const void* q, const void* k,
                            const void* v, void* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  msa_status_t st = check_shape(shape);
  if (st != MSA_OK) return st;
  st = check_seqs(seqs);
  if (st != MSA_OK) return st;
  if (seqs->total_q > 0 && (!q || !k || !v || !out)) return MSA_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, msa_dense_attn_workspace_size(shape, seqs))) return MSA_ERR_WORKSPACE;
  if (cudaMemsetAsync(ws, 0, sizeof(DevError), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (seqs->total_q == 0) return MSA_OK;
  DenseArgs a{};
  a.scratch = static_cast<uint8_t*>(ws) + kWsHeader;
  a.q = q; a.key = k; a.value = v; a.out = out; a.lse = lse;
  a.cu_q = seqs->cu_q; a.cu_k = seqs->cu_k;
  a.batch = seqs->batch; a.H = shape->H; a.G = shape->G; a.d = shape->d; a.sm_scale = shape->sm_scale;
  a.total_q = seqs->total_q; a.total_k = seqs->total_k;
  a.max_q_len = seqs->max_q_len; a.max_k_len = seqs->max_k_len;
  a.err = static_cast<DevError*>(ws);
  return launch_dense_attn(a, stream) == 0 ? MSA_OK : MSA_ERR_CUDA;
}

size_t msa_decode_paged_workspace_size(const msa_shape_t* shape, const msa_paged_t* pages) {
  if (check_paged(shape, pages) != MSA_OK) return 0;
  return paged_layout(shape, pages).total;
}

msa_status_t msa_index_topk_decode_paged(const msa_shape_t* shape, const msa_paged_t* pages, const void* q_idx,
                                         const void* k_idx_pages, int32_t* sel, void* ws, size_t ws_bytes,
                                         void* stream) {
  msa_status_t st = check_paged(shape, pages);
  if (st != MSA_OK) return st;
  if (!q_idx || !k_idx_pages || !sel) return MSA_ERR_INVALID_ARG;
  const PagedLayout L = paged_layout(shape, pages);
  if (!ws_ok(ws, ws_bytes, L.total)) return MSA_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(ws);
  if (cudaMemsetAsync(ws, 0, sizeof(DevError), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MSA_ERR_CUDA;
  int32_t* cu_q = reinterpret_cast<int32_t*>(base + L.cu_q);
  int32_t* cu_k = reinterpret_cast<int32_t*>(base + L.cu_k);
  if (launch_paged_prep(pages->seqlens, pages->batch, pages->max_blocks, cu_q, cu_k, reinterpret_cast<DevError*>(ws),
                        stream) != 0)
    return MSA_ERR_CUDA;
  IndexTopkArgs a{};
  a.q_idx = q_idx; a.k_idx = k_idx_pages; a.sel = sel;
  a.cu_q = cu_q; a.cu_k = cu_k;
  a.batch = pages->batch; a.G = shape->G; a.d_idx = shape->d_idx; a.k = shape->k; a.B_k = kBk;
  a.total_q = pages->batch; a.total_k = L.total_k;
  a.max_q_len = 1; a.max_k_len = pages->max_seqlen;
  a.err = reinterpret_cast<DevError*>(ws);
  a.scratch = base + L.idx_scratch;
  a.scratch_bytes = L.total - L.idx_scratch;
  a.block_table = pages->block_table; a.max_blocks = pages->max_blocks; a.num_pages = pages->num_pages;
  return launch_index_topk_decode(a, stream) == 0 ? MSA_OK : MSA_ERR_CUDA;
}

msa_status_t msa_sparse_attn_decode_paged(const msa_shape_t* shape, const msa_paged_t* pages, const void* q,
                                          const void* k_pages, const void* v_pages, const int32_t* sel, void* out,
                                          float* lse, void* ws, size_t ws_bytes, void* stream) {
  msa_status_t st = check_paged(shape, pages);
  if (st != MSA_OK) return st;
  if (!q || !k_pages || !v_pages || !sel || !out) return MSA_ERR_INVALID_ARG;
  const PagedLayout L = paged_layout(shape, pages);
  if (!ws_ok(ws, ws_bytes, L.total)) return MSA_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(ws);
  if (cudaMemsetAsync(ws, 0, sizeof(DevError), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MSA_ERR_CUDA;
  int32_t* cu_q = reinterpret_cast<int32_t*>(base + L.cu_q);
  int32_t* cu_k = reinterpret_cast<int32_t*>(base + L.cu_k);
  if (launch_paged_prep(pages->seqlens, pages->batch, pages->max_blocks, cu_q, cu_k, reinterpret_cast<DevError*>(ws),
                        stream) != 0)
    return MSA_ERR_CUDA;
  AttnArgs a{};
  a.q = q; a.key = k_pages; a.value = v_pages; a.sel = sel; a.out = out; a.lse = lse;
  a.cu_q = cu_q; a.cu_k = cu_k;
  a.batch = pages->batch; a.H = shape->H; a.G = shape->G; a.d = shape->d; a.k = shape->k; a.B_k = kBk;
  a.sm_scale = shape->sm_scale;
  a.total_q = pages->batch; a.total_k = L.total_k;
  a.max_q_len = 1; a.max_k_len = pages->max_seqlen;
  a.t0 = 0; a.t1 = pages->batch;
  a.err = reinterpret_cast<DevError*>(ws);
  a.tile_ctr = reinterpret_cast<int32_t*>(base + L.tile_ctr);
  a.block_table = pages->block_table; a.max_blocks = pages->max_blocks; a.num_pages = pages->num_pages;
  return launch_rows_attn(a, stream) == 0 ? MSA_OK : MSA_ERR_CUDA;
}

static msa_status_t index_kl_common(const msa_shape_t* shape, const msa_varlen_t* seqs, const void* q, const void* k,
                                   const void* q_idx, const void* k_idx, const int32_t* sel, const float* lse,
                                   float tau, int32_t dense, void* ws, size_t ws_bytes, void* stream,
                                   IndexKlArgs* a) {
  msa_status_t st = check_shape_bk128(shape);
  if (st != MSA_OK) return st;
  st = check_seqs(seqs);
  if (st != MSA_OK) return st;
  if (!(tau == tau) || tau > 3.0e38f || tau < -3.0e38f) return MSA_ERR_INVALID_ARG;   // NaN or infinite
  if (seqs->total_q > 0 && (!q || !k || !q_idx || !k_idx || !lse || (!dense && !sel))) return MSA_ERR_INVALID_ARG;
  // key and index-key rows are read 16 bytes at a time
  if (seqs->total_q > 0 && ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(k_idx)) & 15u))
    return MSA_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, kWsHeader)) return MSA_ERR_WORKSPACE;
  if (cudaMemsetAsync(ws, 0, sizeof(DevError), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MSA_ERR_CUDA;
  a->q = q; a->key = k; a->q_idx = q_idx; a->k_idx = k_idx; a->sel = sel; a->lse = lse;
  a->cu_q = seqs->cu_q; a->cu_k = seqs->cu_k;
  a->batch = seqs->batch; a->H = shape->H; a->G = shape->G; a->d = shape->d; a->d_idx = shape->d_idx;
  a->k = shape->k;
  a->total_q = seqs->total_q;
  a->sm_scale = shape->sm_scale; a->tau = tau; a->dense = dense != 0;
  a->err = static_cast<DevError*>(ws);
  return MSA_OK;
}

// Workspace of the tensor-core KL target, its gradient and the Main Branch
// backward (sparse support): the KV-outer plan of one pass over every query,
// then `tail` bytes (the KL target's float4 partial per (query, group, slot);
// the backward's D per (query, head)).
struct KlLayout {
  size_t blk_off, counts, cursor, tile_sums, nitems, entries, items, part, total;
  int64_t nlists, max_items;
  int32_t qpi, win;
};

size_t kl_part_bytes(const msa_shape_t* s, const msa_varlen_t* v) {
  return sizeof(float4) * (size_t)v->total_q * s->G * s->k;
}

KlLayout kl_layout(const msa_shape_t* s, const msa_varlen_t* v, size_t tail) {
  KlLayout L{};
  const int hg = s->H / s->G;
  const int qpt = 128 / (hg < 8 ? 8 : hg);
  L.qpi = 8 * qpt < kMaxItemQueries ? 8 * qpt : kMaxItemQueries;
  L.nlists = (int64_t)s->G * total_blocks_bound(v, s->B_k);
  L.win = attn_window_rows();
  const int64_t rows = v->total_q;
  const int64_t nkeys = ((rows + L.win - 1) / L.win) * L.nlists;
  const int64_t nentries = rows * s->G * s->k;
  L.max_items = nentries / L.qpi + (nkeys < nentries ? nkeys : nentries) + 1;
  size_t off = kWsHeader;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, kAlign);
    return o;
  };
  L.blk_off = take(sizeof(int32_t) * (v->batch + 1));
  L.counts = take(sizeof(int32_t) * nkeys);
  L.cursor = take(sizeof(int32_t) * nkeys);
  L.tile_sums = take(sizeof(int32_t) * 2 * ((nkeys + kScanTile - 1) / kScanTile + 1));
  L.nitems = take(sizeof(int32_t) * 4);
  L.entries = take(sizeof(uint32_t) * nentries);
  L.items = take(sizeof(Item) * L.max_items);
  L.part = take(tail);
  L.total = off;
  return L;
}

size_t msa_index_kl_workspace_size(const msa_shape_t* shape, const msa_varlen_t* seqs, int32_t dense) {
  if (check_shape_bk128(shape) != MSA_OK || check_seqs(seqs) != MSA_OK) return 0;
  return dense ? kWsHeader : kl_layout(shape, seqs, kl_part_bytes(shape, seqs)).total;
}

// The KV-outer plan of one pass over every query (no query tiles) in the
// workspace of kl_layout.
AttnArgs kl_plan_args(const msa_shape_t* shape, const msa_varlen_t* seqs, const void* q, const void* k,
                      const int32_t* sel, DevError* err, uint8_t* base, const KlLayout& L) {
  AttnArgs p{};
  p.q = q; p.key = k; p.sel = sel;
  p.cu_q = seqs->cu_q; p.cu_k = seqs->cu_k;
  p.batch = seqs->batch; p.H = shape->H; p.G = shape->G; p.d = shape->d; p.k = shape->k; p.B_k = shape->B_k;
  p.sm_scale = shape->sm_scale;
  p.total_q = seqs->total_q; p.total_k = seqs->total_k;
  p.max_q_len = seqs->max_q_len; p.max_k_len = seqs->max_k_len;
  p.t0 = 0; p.t1 = seqs->total_q;
  p.err = err;
  p.blk_off = reinterpret_cast<int32_t*>(base + L.blk_off);
  p.counts = reinterpret_cast<int32_t*>(base + L.counts);
  p.cursor = reinterpret_cast<int32_t*>(base + L.cursor);
  p.tile_sums = reinterpret_cast<int32_t*>(base + L.tile_sums);
  p.nitems = reinterpret_cast<int32_t*>(base + L.nitems);
  p.entries = reinterpret_cast<uint32_t*>(base + L.entries);
  p.items = reinterpret_cast<Item*>(base + L.items);
  p.max_items = L.max_items;
  p.nlists = L.nlists;
  p.win_rows = L.win;
  p.queries_per_item = L.qpi;
  p.theta = 0;
  return p;
}

msa_status_t msa_index_kl(const msa_shape_t* shape, const msa_varlen_t* seqs, const void* q, const void* k,
                          const void* q_idx, const void* k_idx, const int32_t* sel, const float* lse, float tau,
                          int32_t dense, float* kl, float* lse_z, void* ws, size_t ws_bytes, void* stream) {
  if (seqs != nullptr && seqs->total_q > 0 && kl == nullptr) return MSA_ERR_INVALID_ARG;
  IndexKlArgs a{};
  const msa_status_t st = index_kl_common(shape, seqs, q, k, q_idx, k_idx, sel, lse, tau, dense, ws, ws_bytes,
                                          stream, &a);
  if (st != MSA_OK || seqs->total_q == 0) return st;
  a.kl = kl;
  a.lse_z = lse_z;
  if (dense) return launch_index_kl(a, stream) == 0 ? MSA_OK : MSA_ERR_CUDA;
  // selected support: the tensor-core form over the forward's KV-outer lists
  // (its index-query rows are read 16 bytes at a time)
  if (reinterpret_cast<uintptr_t>(q_idx) & 15u) return MSA_ERR_INVALID_ARG;
  const KlLayout L = kl_layout(shape, seqs, kl_part_bytes(shape, seqs));
  if (!ws_ok(ws, ws_bytes, L.total)) return MSA_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(ws);
  const AttnArgs p = kl_plan_args(shape, seqs, q, k, sel, a.err, base, L);
  return launch_index_kl_tc(a, p, reinterpret_cast<float4*>(base + L.part), stream) == 0 ? MSA_OK : MSA_ERR_CUDA;
}

msa_status_t msa_index_kl_backward(const msa_shape_t* shape, const msa_varlen_t* seqs, const void* q,
                                   const void* k, const void* q_idx, const void* k_idx, const int32_t* sel,
                                   const float* lse, const float* lse_z, float tau, int32_t dense, float* dq_idx,
                                   float* dk_idx, void* ws, size_t ws_bytes, void* stream) {
  if (seqs != nullptr && seqs->total_q > 0 && (lse_z == nullptr || dq_idx == nullptr || dk_idx == nullptr))
    return MSA_ERR_INVALID_ARG;
  // the index-key gradient's rows are added 16 bytes at a time
  if (seqs != nullptr && seqs->total_q > 0 && (reinterpret_cast<uintptr_t>(dk_idx) & 15u))
    return MSA_ERR_INVALID_ARG;
  IndexKlArgs a{};
  const msa_status_t st = index_kl_common(shape, seqs, q, k, q_idx, k_idx, sel, lse, tau, dense, ws, ws_bytes,
                                          stream, &a);
  if (st != MSA_OK || seqs->total_q == 0) return st;
  // selected support: the tensor-core form over the same plan as msa_index_kl
  // (index-query rows read and dq_idx rows added 16 bytes at a time)
  KlLayout L{};
  if (!dense) {
    if ((reinterpret_cast<uintptr_t>(q_idx) | reinterpret_cast<uintptr_t>(dq_idx)) & 15u)
      return MSA_ERR_INVALID_ARG;
    L = kl_layout(shape, seqs, kl_part_bytes(shape, seqs));
    if (!ws_ok(ws, ws_bytes, L.total)) return MSA_ERR_WORKSPACE;
  }
  // the key gradient is accumulated over every query that reaches a key row
  if (cudaMemsetAsync(dk_idx, 0, sizeof(float) * (size_t)seqs->total_k * shape->d_idx,
                      reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MSA_ERR_CUDA;
  a.lse_z = const_cast<float*>(lse_z);
  a.dq_idx = dq_idx;
  a.dk_idx = dk_idx;
  if (dense) return launch_index_kl_backward(a, stream) == 0 ? MSA_OK : MSA_ERR_CUDA;
  const AttnArgs p = kl_plan_args(shape, seqs, q, k, sel, a.err, static_cast<uint8_t*>(ws), L);
  return launch_index_kl_grad_tc(a, p, stream) == 0 ? MSA_OK : MSA_ERR_CUDA;
}

msa_status_t msa_select_window(const msa_shape_t* shape, const msa_varlen_t* seqs, int32_t n_sink, int32_t* sel,
                               void* ws, size_t ws_bytes, void* stream) {
  msa_status_t st = check_shape_bk128(shape);
  if (st != MSA_OK) return st;
  st = check_seqs(seqs);
  if (st != MSA_OK) return st;
  if (n_sink < 0 || n_sink >= shape->k) return MSA_ERR_INVALID_ARG;
  if (seqs->total_q > 0 && sel == nullptr) return MSA_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, kWsHeader)) return MSA_ERR_WORKSPACE;
  if (cudaMemsetAsync(ws, 0, sizeof(DevError), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (seqs->total_q == 0) return MSA_OK;
  return launch_window_select(seqs->cu_q, seqs->cu_k, seqs->batch, shape->G, shape->k, n_sink, seqs->total_q, sel,
                              static_cast<DevError*>(ws), stream) == 0
             ? MSA_OK
             : MSA_ERR_CUDA;
}

size_t msa_sparse_attn_backward_workspace_size(const msa_shape_t* shape, const msa_varlen_t* seqs, int32_t dense) {
  if (check_shape_bk128(shape) != MSA_OK || check_seqs(seqs) != MSA_OK) return 0;
  return dense ? kWsHeader : kl_layout(shape, seqs, sizeof(float) * (size_t)seqs->total_q * shape->H).total;
}

msa_status_t msa_sparse_attn_backward(const msa_shape_t* shape, const msa_varlen_t* seqs, const void* q,
                                      const void* k, const void* v, const int32_t* sel, const void* out,
                                      const float* lse, const void* dout, int32_t dense, float* dq, float* dk,
                                      float* dv, void* ws, size_t ws_bytes, void* stream) {
  msa_status_t st = check_shape_bk128(shape);
  if (st != MSA_OK) return st;
  st = check_seqs(seqs);
  if (st != MSA_OK) return st;
  if (seqs->total_q > 0 &&
      (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv || (!dense && !sel)))
    return MSA_ERR_INVALID_ARG;
  // key / value rows are read, and dk / dv rows added, 16 bytes at a time;
  // the selected support also reads out / dout rows and adds dq rows so
  if (seqs->total_q > 0 && ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) |
                             reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv)) & 15u))
    return MSA_ERR_INVALID_ARG;
  if (seqs->total_q > 0 && !dense &&
      ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out) | reinterpret_cast<uintptr_t>(dout) |
        reinterpret_cast<uintptr_t>(dq)) & 15u))
    return MSA_ERR_INVALID_ARG;
  const KlLayout L = kl_layout(shape, seqs, sizeof(float) * (size_t)seqs->total_q * shape->H);
  if (!ws_ok(ws, ws_bytes, dense ? kWsHeader : L.total)) return MSA_ERR_WORKSPACE;
  cudaStream_t st_ = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(DevError), st_) != cudaSuccess) return MSA_ERR_CUDA;
  if (seqs->total_q == 0) return MSA_OK;
  // dk and dv are accumulated over every query that reaches a key row
  const size_t kv_bytes = sizeof(float) * (size_t)seqs->total_k * shape->G * shape->d;
  if (cudaMemsetAsync(dk, 0, kv_bytes, st_) != cudaSuccess || cudaMemsetAsync(dv, 0, kv_bytes, st_) != cudaSuccess)
    return MSA_ERR_CUDA;
  AttnBwdArgs a{};
  a.q = q; a.key = k; a.value = v; a.sel = sel; a.out = out; a.lse = lse; a.dout = dout;
  a.cu_q = seqs->cu_q; a.cu_k = seqs->cu_k;
  a.batch = seqs->batch; a.H = shape->H; a.G = shape->G; a.d = shape->d; a.k = shape->k;
  a.total_q = seqs->total_q;
  a.sm_scale = shape->sm_scale; a.dense = dense != 0;
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.err = static_cast<DevError*>(ws);
  if (dense) return launch_sparse_attn_backward(a, stream) == 0 ? MSA_OK : MSA_ERR_CUDA;
  // selected support: the tensor-core form over the forward's KV-outer lists
  uint8_t* base = static_cast<uint8_t*>(ws);
  const AttnArgs p = kl_plan_args(shape, seqs, q, k, sel, a.err, base, L);
  return launch_sparse_attn_backward_tc(a, p, reinterpret_cast<float*>(base + L.part), stream) == 0 ? MSA_OK
                                                                                                       : MSA_ERR_CUDA;
}

msa_status_t msa_selected_share(const float* lse_sel, const float* lse_all, int64_t n, float* share, void* stream) {
  if (n < 0) return MSA_ERR_INVALID_ARG;
  if (n > 0 && (!lse_sel || !lse_all || !share)) return MSA_ERR_INVALID_ARG;
  return launch_selected_share(lse_sel, lse_all, n, share, stream) == 0 ? MSA_OK : MSA_ERR_CUDA;
}

msa_status_t msa_index_topk_policy(const msa_shape_t* shape, const msa_varlen_t* seqs, int32_t n_sink,
                                   int32_t n_local, const void* q_idx, const void* k_idx, int32_t* sel, void* ws,
                                   size_t ws_bytes, void* stream) {
  msa_status_t st = check_shape_bk128(shape);
  if (st != MSA_OK) return st;
  st = check_seqs(seqs);
  if (st != MSA_OK) return st;
  if (n_sink < 0 || n_local < 1 || n_sink + n_local > shape->k) return MSA_ERR_INVALID_ARG;
  if ((int64_t)seqs->max_k_len > (int64_t)8192 * kBk) return MSA_ERR_UNSUPPORTED;   // block scores in shared memory
  if (seqs->total_q > 0 && (!q_idx || !k_idx || !sel)) return MSA_ERR_INVALID_ARG;
  // index-key rows are read 16 bytes at a time
  if (seqs->total_q > 0 && (reinterpret_cast<uintptr_t>(k_idx) & 15u)) return MSA_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, kWsHeader)) return MSA_ERR_WORKSPACE;
  if (cudaMemsetAsync(ws, 0, sizeof(DevError), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (seqs->total_q == 0) return MSA_OK;
  return launch_policy_select(q_idx, k_idx, seqs->cu_q, seqs->cu_k, seqs->batch, shape->G, shape->d_idx, shape->k,
                              n_sink, n_local, seqs->total_q, sel, static_cast<DevError*>(ws), stream) == 0
             ? MSA_OK
             : MSA_ERR_CUDA;
}

msa_status_t msa_gather_pages(const msa_varlen_t* seqs, const int32_t* block_table, int32_t max_blocks,
                              int64_t num_pages, int64_t row_bytes, const void* pages, void* packed, void* ws,
                              size_t ws_bytes, void* stream) {
  if (seqs == nullptr || seqs->cu_k == nullptr || seqs->batch < 1 || seqs->max_k_len < 0 || seqs->total_k < 0)
    return MSA_ERR_INVALID_ARG;
  if (block_table == nullptr || max_blocks < 1 || num_pages < 1) return MSA_ERR_INVALID_ARG;
  if ((int64_t)seqs->max_k_len > (int64_t)max_blocks * kBk) return MSA_ERR_INVALID_ARG;
  if (row_bytes <= 0 || row_bytes % 16 != 0) return MSA_ERR_INVALID_ARG;
  if (seqs->total_k > 0 &&
      (!pages || !packed || ((reinterpret_cast<uintptr_t>(pages) | reinterpret_cast<uintptr_t>(packed)) & 15u)))
    return MSA_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, kWsHeader)) return MSA_ERR_WORKSPACE;
  if (cudaMemsetAsync(ws, 0, sizeof(DevError), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (seqs->total_k == 0) return MSA_OK;
  return launch_gather_pages(seqs->cu_k, seqs->batch, seqs->max_k_len, block_table, max_blocks, num_pages, row_bytes,
                             pages, packed, static_cast<DevError*>(ws), stream) == 0
             ? MSA_OK
             : MSA_ERR_CUDA;
}

int32_t msa_set_tile_threshold(int32_t theta) {
  return g_tile_theta.exchange(theta < 0 ? -1 : theta);
}

int32_t msa_set_attn_window(int32_t rows) {
  if (rows <= 0) rows = kDefaultWindow;
  if (rows < kMinWindow) rows = kMinWindow;
  if (rows > kMaxWindow) rows = kMaxWindow;
  return g_attn_window.exchange(rows);
}

msa_status_t msa_get_device_error(void* ws, int32_t* code, int32_t* where, int32_t* info0, int32_t* info1,
                                  void* stream) {
  if (ws == nullptr || code == nullptr) return MSA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DevError h{};
  if (cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return MSA_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(h), st) != cudaSuccess) return MSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MSA_ERR_CUDA;
  *code = h.code;
  if (where) *where = h.where;
  if (info0) *info0 = h.info0;
  if (info1) *info1 = h.info1;
  return MSA_OK;
}

}  // extern "C"
