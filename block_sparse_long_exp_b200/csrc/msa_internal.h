// Definitions shared by the host-side API and the kernels of libmsa.
#pragma once

#include <stddef.h>
#include <stdint.h>
#include <vector_types.h>

#include "../../include/msa.h"

namespace msa {

constexpr int kBk = 128;          // key tile of the kernels (the largest block size B_k; 32 and 64 divide it)
constexpr int kMaxK = 32;         // largest k
constexpr int kMaxBatchTiles = 1024;  // sequences per prefill index launch
constexpr int kDefaultWindow = 8192;  // query rows per attention planning window (KV-outer lists)
constexpr int kMinWindow = 128;
constexpr int kMaxWindow = 1 << 20;
constexpr int kScanTile = 4096;       // keys per CTA of the planning scan
constexpr int kMaxItemQueries = 64;   // queries per attention work item (upper bound)
constexpr int kMaxDense = 64;         // dense blocks per query tile (Q-outer side)
constexpr int32_t kDenseComplete = 1;   // dstate: the tile covers every selection of the query

// Device error word, at offset 0 of every workspace.
struct DevError {
  int32_t code;
  int32_t where;
  int32_t info0;
  int32_t info1;
};

// Sites that can record an error (DevError::where).
enum ErrorSite : int32_t {
  kSiteIndexProducer = 101,
  kSiteIndexMma = 102,
  kSiteIndexEpilogue = 103,
  kSiteIndexSeq = 104,
  kSiteDecodeIndex = 111,
  kSiteInvert = 121,
  kSiteAttnLoad = 131,
  kSiteAttnMma = 132,
  kSiteAttnSoftmax = 133,
  kSiteAttnItem = 134,
  kSiteDense = 141,
  kSiteTileUnit = 151,
  kSiteTileLoad = 152,
  kSiteTileMma = 153,
  kSiteTileSoftmax = 154,
  kSitePaged = 161,
  kSiteSelfTest = 221,
  kSiteKeySplit = 231,
};

// One KV-outer work item: up to `count` queries of the list of
// (sequence seq, group g, block blk), entries [start, start + count) of the
// packed query lists.
struct Item {
  int32_t seq;
  int32_t blk;
  int32_t g;
  int32_t start;
  int32_t count;
  int32_t pad0, pad1, pad2;
};

constexpr size_t kWsHeader = 256;  // DevError + counters

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Host-side argument checks shared by the entry points (msa_api.cu).
msa_status_t check_shape(const msa_shape_t* s);
msa_status_t check_shape_bk128(const msa_shape_t* s);
msa_status_t check_seqs(const msa_varlen_t* v);

// -------------------------------------------------------- host launchers ---
// Each returns the cudaError_t of its launch(es) (0 on success).

struct IndexTopkArgs {
  const void* q_idx;   // bf16 [T, G, d_idx]
  const void* k_idx;   // bf16 [S, d_idx]
  int32_t* sel;        // [T, G, k]
  const int32_t* cu_q;
  const int32_t* cu_k;
  int32_t batch, G, d_idx, k;
  int32_t B_k;         // block size: 32, 64 or 128 (a divisor of the 128-key tile)
  int32_t all_blocks;  // decode: the query lies after the keys (every complete block is scored)
  float* cand_score;   // decode: non-null -> write the k-1 candidates (ids in sel [T, G, k-1]) and their scores
  int64_t total_q, total_k;
  int32_t max_q_len, max_k_len;
  DevError* err;
  void* scratch;       // decode path: block scores
  size_t scratch_bytes;
  // paged caches (decode): block j of sequence b is page block_table[b * max_blocks + j]
  const int32_t* block_table;   // null: packed rows cu_k[b] + j * B_k
  int32_t max_blocks;
  int64_t num_pages;
  // prefill: the 128-query tiles whose first row lies in [row0, row1) (row1 <= 0: total_q),
  // on `grid` CTAs (<= 0: one per SM)
  int64_t row0, row1;
  int32_t grid;
};
int launch_index_topk_prefill(const IndexTopkArgs& a, void* stream);
int launch_index_topk_decode(const IndexTopkArgs& a, void* stream);
size_t decode_index_scratch_bytes(int32_t batch, int64_t total_k, int32_t G, int32_t B_k);

struct AttnArgs {
  const void* q;       // bf16 [T, H, d]
  const void* key;     // bf16 [S, G, d]
  const void* value;   // bf16 [S, G, d]
  const int32_t* sel;  // [T, G, k]
  void* out;           // bf16 [T, H, d]
  float* lse;          // [T, H] or null
  const int32_t* cu_q;
  const int32_t* cu_k;
  int32_t batch, H, G, d, k;
  int32_t B_k;         // block size: 32, 64 or 128
  float sm_scale;
  int64_t total_q, total_k;
  int32_t max_q_len, max_k_len;
  int64_t t0, t1;      // query rows of this pass
  DevError* err;
  // workspace slices
  int32_t* counts;     // [nwin * nlists]  entries per (window, list)
  int32_t* cursor;     // [nwin * nlists]  list offsets, then scatter cursors
  int32_t* tile_sums;  // [2 * ceil(nwin * nlists / kScanTile)]
  int32_t* nitems;     // [4]: items, item ticket, entries
  uint32_t* entries;   // [(t1 - t0) * G * k]
  Item* items;         // [max_items]
  int64_t max_items;
  int32_t* blk_off;    // [batch + 1] block offsets per sequence
  int64_t nlists;      // G * total blocks
  int32_t win_rows;    // query rows per planning window (lists are keyed by (group, window, block))
  void* part_acc;      // f16 [(t1-t0), G, k, d/8, Hg, 8], each pair's partials packed at slots 0..n-1
  float* part_lse;     // [(t1-t0), G, k, Hg]
  int32_t queries_per_item;
  // query-tile (Q-outer) side; theta == 0 turns it off
  int32_t theta;       // a block is a tile's dense block when >= theta of its queries chose it
  int32_t* unit_blk;   // [units x G][kMaxDense]
  int32_t* unit_nblk;  // [units x G]
  int32_t* unit_list;  // [units x G] units with dense blocks
  uint32_t* dmask;     // [(t1-t0) x G] slots covered by the tile
  int32_t* dstate;     // [(t1-t0) x G] -1: no slot covered; 0: some; kDenseComplete: all
  uint64_t* dmember;   // [(t1-t0) x G] positions of the covered blocks in the tile's list
  uint2* clist;        // [(t1-t0) x G] combine list: {pair (t - t0) * G + g, slots to merge}
  int32_t* tile_ctr;   // [4]: pairs, listed units, unit ticket
  // paged caches (decode, rows mode): see IndexTopkArgs
  const int32_t* block_table;
  int32_t max_blocks;
  int64_t num_pages;
};
int launch_sparse_attn_pass(const AttnArgs& a, void* stream);   // main phase, then the combine
// The two phases of a pass on their own: the main phase (planning, lists,
// KV-outer and query-tile attention) writes the pass's partials; the combine
// merges them into out / lse (on at most grid_cap CTAs; <= 0: one per SM).
int launch_sparse_attn_main(const AttnArgs& a, void* stream);
// The planning of a pass alone (block offsets, the query-tile plan when theta
// > 0, the KV-outer lists and their work items); launch_sparse_attn_main runs
// it first.
int launch_kv_plan(const AttnArgs& a, void* stream);
int launch_sparse_attn_combine(const AttnArgs& a, void* stream, int grid_cap);
int attn_window_rows();                // planning window of the prefill calls (msa_set_attn_window)
int launch_combine(const void* part_acc, const float* part_lse, const int32_t* sel, void* out,
                   float* lse, int64_t T, int32_t H, int32_t G, int32_t d, int32_t k, void* stream);
int tile_queries(int H, int G);        // query rows per tile unit
int tile_default_theta(int UQ);
int launch_tile_plan(const AttnArgs& a, int theta, void* stream);
int launch_tile_attn(const AttnArgs& a, void* stream);
int launch_rows_attn(const AttnArgs& a, void* stream);   // one query per unit (decode)
// Paged decode: cu_q[b] = b and cu_k = prefix of seqlens (a length outside
// [1, max_blocks * B_k] counts as 0 and records MSA_ERR_DEVICE_CHECK).
int launch_paged_prep(const int32_t* seqlens, int32_t batch, int32_t max_blocks, int32_t* cu_q, int32_t* cu_k,
                      DevError* err, void* stream);

struct DenseArgs {
  const void* q;
  const void* key;
  const void* value;
  void* out;
  float* lse;
  const int32_t* cu_q;
  const int32_t* cu_k;
  int32_t batch, H, G, d;
  float sm_scale;
  int64_t total_q, total_k;
  int32_t max_q_len, max_k_len;
  DevError* err;
  void* scratch;       // dense_scratch_bytes(batch)
};
size_t dense_scratch_bytes(int32_t batch);
int launch_dense_attn(const DenseArgs& a, void* stream);

// Launch accounting: a ProfScope wraps one kernel launch; it always counts the
// launch and, while profiling is enabled (msa_profile_enable), records a CUDA
// event pair around it on the launch stream.
void prof_count_launch(int n);
class ProfScope {
 public:
  ProfScope(const char* name, void* stream);
  ~ProfScope();
  ProfScope(const ProfScope&) = delete;
  ProfScope& operator=(const ProfScope&) = delete;

 private:
  const char* name_;
  void* stream_;
  void* start_;
  void* stop_;
};

// Tensor-map creation (driver entry point resolved at run time).
int make_tmap_bf16(void* tmap_out, const void* base, int rank, const uint64_t* dims,
                   const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes);

}  // namespace msa
