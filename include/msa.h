/*
 * msa.h — C ABI of the MiniMax Sparse Attention (MSA) forward hot path on
 * NVIDIA B200 (sm_100a).  Library: libmsa.so.
 *
 * The operation (web pages on MSA, cited by title / address and section):
 *   - pnsm.cn explainer "MiniMax Sparse Attention：一篇读懂百万上下文时代的稀疏注意力
 *     工程化路线", sec. 2 (group-specific block selection on GQA, local block
 *     always kept, B_k = 128, k = 16) and sec. 7 (exp-free Top-k, KV-outer
 *     sparse attention, query gather, two-phase combine, load balancing);
 *   - yifor-blog "MiniMax Sparse Attention (MSA): a Two-Branch Block-Sparse
 *     Attention ...", section "設計核心" (Index Branch: block scores by
 *     max-pooling, top-k; Main Branch: exact softmax on the chosen blocks);
 *   - yhxrc.cn article, sec. 二 "MSA是怎么做的" (one index query head per group
 *     and one shared index key head; current block mandatory; KV-outer).
 *
 * Conventions shared by every entry point
 *   - All pointers named as device pointers must point to device memory of
 *     the current CUDA device; the caller owns every buffer.  The library
 *     allocates nothing: its scratch space is the caller's workspace `ws`
 *     (size from the matching *_workspace_size query, 256-byte aligned).
 *   - Every call is asynchronous on `stream` (a cudaStream_t, 0 = legacy
 *     default stream).  Calls that share a workspace must be ordered.
 *   - Tensors are contiguous, row-major, bf16 unless stated:
 *       q      [T, H, d]        query heads of every query token
 *       k, v   [S, G, d]        keys / values (G = KV heads = GQA groups)
 *       q_idx  [T, G, d_idx]    index query: one head per group
 *       k_idx  [S, d_idx]       index key: one head shared by all groups
 *       sel    [T, G, k] int32  selected block ids (local to the sequence),
 *                               ascending, padded with -1
 *       out    [T, H, d]        attention output
 *       lse    [T, H] float     natural-log log-sum-exp of the scaled scores
 *   - Sequences are packed: sequence b owns query rows cu_q[b]..cu_q[b+1]-1
 *     and key rows cu_k[b]..cu_k[b+1]-1 (int32 device arrays of batch+1).
 *     Its queries are its LAST T_b = cu_q[b+1]-cu_q[b] tokens: query i sits at
 *     position S_b - T_b + i (prefill: T_b = S_b; decode: T_b = 1).
 *     T_b <= S_b is required (checked on the device: MSA_ERR_DEVICE_CHECK).
 *   - Query head h belongs to group g = h / (H / G).
 *   - Block j of a sequence holds its tokens [j*B_k, (j+1)*B_k).  A query at
 *     position p has local block lb = p / B_k and attends causally (keys <= p).
 *   - Selection rule: the local block always; the other k-1 blocks are the
 *     best of blocks 0..lb-1 by block score (max over the block's tokens of
 *     <q_idx[t,g], k_idx[j]>), ties to the lower block index; NaN scores rank
 *     as -inf; with lb+1 <= k all causal blocks are selected.
 *
 * Errors
 *   - Arguments are checked on the host before any launch: MSA_ERR_INVALID_ARG
 *     (null pointer, bad size), MSA_ERR_UNSUPPORTED (a size the kernels are not
 *     built for), MSA_ERR_WORKSPACE (ws too small or misaligned).  Nothing is
 *     launched when a check fails.
 *   - A launch failure returns MSA_ERR_CUDA (cudaGetLastError after launch).
 *   - Kernels record data-dependent failures (a bounded wait that ran out, a
 *     block id out of range, T_b > S_b) in an error word at the start of `ws`.
 *     Each call clears the word when it starts; read it with
 *     msa_get_device_error after the call (it waits for the stream).
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A call with no queries (total_q == 0; T == 0 for msa_combine) launches
 * nothing and returns MSA_OK after the argument checks; its data pointers may
 * then be NULL (empty tensors need no storage).  The workspace rules still
 * apply and its error word is cleared. */
typedef enum {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1,
  MSA_ERR_UNSUPPORTED = 2,
  MSA_ERR_WORKSPACE = 3,
  MSA_ERR_CUDA = 4,
  MSA_ERR_TIMEOUT = 5,
  MSA_ERR_DEVICE_CHECK = 6
} msa_status_t;

/* Layer shape.  Supported: H % G == 0 with H/G in {4, 8, 16}; G in {1, 2, 4};
 * d in {64, 128}; d_idx in {32, 64, 128}; B_k == 128; 1 <= k <= 32. */
typedef struct {
  int32_t H;        /* query heads */
  int32_t G;        /* KV heads = GQA groups = index query heads */
  int32_t d;        /* head dim of q / k / v */
  int32_t d_idx;    /* index head dim */
  int32_t B_k;      /* block size in tokens */
  int32_t k;        /* blocks selected per (query, group), local block included */
  float sm_scale;   /* main-branch softmax scale (usually 1/sqrt(d)) */
} msa_shape_t;

/* Packed-sequence description.  cu_q / cu_k are DEVICE pointers; the other
 * fields are host values that must agree with them: total_q = cu_q[batch],
 * total_k = cu_k[batch], max_q_len / max_k_len the largest T_b / S_b, and
 * cu_q[0] = cu_k[0] = 0 with both non-decreasing.  The library sizes its
 * launches and buffers from the host values and does not read the device
 * arrays back (that would synchronise the stream), so this agreement is the
 * caller's to keep: offsets beyond total_q / total_k make kernels read and
 * write outside the caller's buffers.  T_b > S_b is checked on the device
 * (MSA_ERR_DEVICE_CHECK).  The Python binding checks the host copies. */
typedef struct {
  int32_t batch;
  int32_t max_q_len;
  int32_t max_k_len;
  int32_t pad_;
  int64_t total_q;
  int64_t total_k;
  const int32_t* cu_q;
  const int32_t* cu_k;
} msa_varlen_t;

/* ---------------------------------------------------------------------- */
/* Index Branch: block scoring + top-k with the forced local block.
 * (pnsm.cn sec. 2 and sec. 7 "exp-free Top-k"; yifor-blog "設計核心" item 1;
 *  yhxrc.cn sec. 二 "block max pooling".)
 *
 * Scores every causal, non-local block of every (query, group) with raw dot
 * products (no exp), max-pools them per block and writes the selection
 * sel[T, G, k].  Prefill-shaped calls (max_q_len > 1) run a tensor-core
 * kernel over 128-query tiles; decode-shaped calls (max_q_len == 1) run a
 * split scan of the index keys and a candidate merge.
 * Selections are exact for inputs whose scores are exact in fp32 (for
 * example integer-valued index q/k); otherwise they follow fp32 rounding.
 * Prefill-shaped calls take at most 1024 sequences (MSA_ERR_UNSUPPORTED
 * beyond, and the workspace query returns 0); decode-shaped calls have no
 * such limit. */
size_t msa_index_topk_workspace_size(const msa_shape_t* shape, const msa_varlen_t* seqs);

msa_status_t msa_index_topk(const msa_shape_t* shape, const msa_varlen_t* seqs,
                            const void* q_idx,  /* device bf16 [T, G, d_idx] */
                            const void* k_idx,  /* device bf16 [S, d_idx] */
                            int32_t* sel,       /* device int32 [T, G, k] (out) */
                            void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* Main Branch, prefill: exact causal softmax attention over the selected
 * blocks (yifor-blog "設計核心" item 2; yololab.net "MSA的兩個主要步驟" step 2),
 * computed KV-outer (pnsm.cn sec. 7; yhxrc.cn sec. 二; yololab.net "KV Outer
 * Gather Q"): the selection is inverted into per-(sequence, group, block)
 * query lists, each KV block is loaded once per work item and every query that
 * chose it is gathered into tensor-core tiles; each (query, group, block)
 * writes a softmax partial that a log-sum-exp combine merges (two-phase
 * combine, no atomics on the output).
 *
 * `q_chunk` bounds how many query rows are processed per pass (0 = all); the
 * workspace grows with it (about G*k*(H/G)*(2d+4) bytes per query row).  The
 * call loops over chunks itself.  `lse` may be NULL. */
size_t msa_sparse_attn_workspace_size(const msa_shape_t* shape, const msa_varlen_t* seqs,
                                      int64_t q_chunk);

msa_status_t msa_sparse_attn_prefill(const msa_shape_t* shape, const msa_varlen_t* seqs,
                                     const void* q,       /* device bf16 [T, H, d] */
                                     const void* k,       /* device bf16 [S, G, d] */
                                     const void* v,       /* device bf16 [S, G, d] */
                                     const int32_t* sel,  /* device int32 [T, G, k] */
                                     void* out,           /* device bf16 [T, H, d] (out) */
                                     float* lse,          /* device f32 [T, H] (out) or NULL */
                                     int64_t q_chunk,
                                     void* ws, size_t ws_bytes, void* stream);

/* One MSA layer, prefill: the Index Branch and the Main Branch of the same
 * layer in one call (pnsm.cn sec. 2: block scoring and top-k select the
 * blocks, then block-sparse attention runs over them; yololab.net
 * "MSA的兩個主要步驟").  Writes the selection `sel` exactly as msa_index_topk
 * and `out` / `lse` exactly as msa_sparse_attn_prefill with the same q_chunk
 * (bit for bit: every row is computed by the same kernels in the same order).
 *
 * The work runs in passes of q_chunk query rows (0 = all rows in one pass).
 * For each pass: the index top-k of the 128-query tiles whose first row lies
 * in the pass, then the pass's attention.  With more than one pass the
 * library overlaps the combine of pass p (memory-bound) with the index top-k
 * of pass p + 1 (compute-bound, few DRAM bytes): the combine runs on a second
 * stream of the library's own, on the SMs set by msa_set_prefill_overlap, the
 * index kernel on the others; events order the two streams, and when the call
 * returns everything it enqueued is ordered before later work on `stream`.
 * Calls from several host threads serialize their enqueue on one lock.  The
 * second stream and its two events are created by the first overlapped call on
 * a device and kept for the life of the process (a cudaDeviceReset ends their
 * use on that device: later overlapped calls there return MSA_ERR_CUDA).  The
 * overlap is off by default: measured on B200 at 128K tokens, a combine on 16
 * to 48 of the 148 SMs is bound by its own latency and outlasts the index pass
 * it hides behind (the step got 3-20 ms slower), so every pass runs on the
 * caller's stream over all SMs unless msa_set_prefill_overlap asks otherwise.
 *
 * q_idx / k_idx as msa_index_topk, q / k / v / out / lse as
 * msa_sparse_attn_prefill.  Prefill shapes only (max_q_len > 1; decode has its
 * own calls) and at most 1024 sequences.  Workspace: one block of
 * msa_prefill_workspace_size bytes (256-byte aligned); its error word reports
 * both branches' device checks. */
size_t msa_prefill_workspace_size(const msa_shape_t* shape, const msa_varlen_t* seqs, int64_t q_chunk);

msa_status_t msa_prefill(const msa_shape_t* shape, const msa_varlen_t* seqs,
                         const void* q,      /* device bf16 [T, H, d] */
                         const void* k,      /* device bf16 [S, G, d] */
                         const void* v,      /* device bf16 [S, G, d] */
                         const void* q_idx,  /* device bf16 [T, G, d_idx] */
                         const void* k_idx,  /* device bf16 [S, d_idx] */
                         int32_t* sel,       /* device int32 [T, G, k] (out) */
                         void* out,          /* device bf16 [T, H, d] (out) */
                         float* lse,         /* device f32 [T, H] (out) or NULL */
                         int64_t q_chunk,
                         void* ws, size_t ws_bytes, void* stream);

/* SMs that msa_prefill gives the combine of a pass while the next pass's
 * index top-k runs on the rest; returns the previous value.
 *   sms < 0     the default (0)
 *   sms == 0    no overlap: every kernel of the call runs on the caller's
 *               stream over all SMs
 *   otherwise   at most half of the device's SMs
 * Results do not depend on it.  One atomic word, read once per call. */
int32_t msa_set_prefill_overlap(int32_t sms);

/* Main Branch, decode: one query per sequence (T_b = 1, position S_b - 1,
 * the cache already holding the new token), the decode step of pnsm.cn
 * sec. 9 and yhxrc.cn sec. 二.  Same contract as the prefill call; q_chunk
 * is implied (all queries in one pass). */
msa_status_t msa_sparse_attn_decode(const msa_shape_t* shape, const msa_varlen_t* seqs,
                                    const void* q, const void* k_cache, const void* v_cache,
                                    const int32_t* sel, void* out, float* lse,
                                    void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* Decode over a paged KV cache (a serving layout; the pages describe the
 * method, not a cache format, and this is the plainest paged form of their
 * decode step: pnsm.cn sec. 9, yhxrc.cn sec. 二).  A page holds one B_k-token
 * block: page p is rows [p*B_k, (p+1)*B_k) of
 *   k_idx_pages  device bf16 [num_pages*B_k, d_idx]
 *   k_pages      device bf16 [num_pages*B_k, G, d]
 *   v_pages      device bf16 [num_pages*B_k, G, d]
 * Sequence b holds seqlens[b] tokens (the new token included, so its one
 * query sits at position seqlens[b]-1); its block j lives in page
 * block_table[b*max_blocks + j] for j < ceil(seqlens[b]/B_k).  Token rows
 * past seqlens[b] in the last page are never attended.  q / q_idx / sel /
 * out / lse have one row per sequence ([batch, ...], as in the packed decode
 * call).  Results equal those of the packed calls on the same tokens. */
typedef struct {
  int32_t batch;
  int32_t max_blocks;        /* columns of block_table */
  int32_t max_seqlen;        /* host upper bound of seqlens[b] */
  int32_t pad_;
  int64_t num_pages;
  const int32_t* seqlens;    /* device [batch] */
  const int32_t* block_table;/* device [batch, max_blocks] */
} msa_paged_t;

/* Workspace of either paged call (the same size serves both). */
size_t msa_decode_paged_workspace_size(const msa_shape_t* shape, const msa_paged_t* pages);

/* Index branch over the paged index keys: sel [batch, G, k] as
 * msa_index_topk.  A page id outside [0, num_pages) or seqlens[b] outside
 * [1, max_blocks*B_k] records MSA_ERR_DEVICE_CHECK in the error word (the
 * sequence is skipped; nothing is read out of range). */
msa_status_t msa_index_topk_decode_paged(const msa_shape_t* shape, const msa_paged_t* pages,
                                         const void* q_idx, const void* k_idx_pages, int32_t* sel,
                                         void* ws, size_t ws_bytes, void* stream);

/* Main branch over the paged K / V: out [batch, H, d] (and lse [batch, H] or
 * NULL) from the selection sel [batch, G, k].  Same device checks. */
msa_status_t msa_sparse_attn_decode_paged(const msa_shape_t* shape, const msa_paged_t* pages,
                                          const void* q, const void* k_pages, const void* v_pages,
                                          const int32_t* sel, void* out, float* lse,
                                          void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* Prefill (or a chunk of one) over a paged KV cache: gather the pages into
 * packed rows, then run the packed calls.  The pages give no cache format.
 * lumevalley.com says MSA on GQA keeps a serving stack's existing KV-cache
 * management and replaces only the attention kernel; this is the plainest
 * way to take such a cache into the prefill.  Packed row cu_k[b] + j of sequence
 * b is row (p * B_k + j mod B_k) of `pages`, p = block_table[b * max_blocks +
 * j / B_k]; rows are row_bytes each (a multiple of 16; index keys: d_idx * 2,
 * keys or values: G * d * 2).  seqs gives the lengths (cu_k, max_k_len <=
 * max_blocks * B_k); pages holds num_pages * B_k rows and packed total_k rows,
 * both 16-byte aligned.  A page outside [0, num_pages) is recorded as
 * MSA_ERR_DEVICE_CHECK and its rows are written as zeros.  ws: at least 256
 * bytes, 256-byte aligned.  The gather is one extra pass over the rows (HBM
 * bound); the results of the packed calls on its output are those of the
 * same calls on the same tokens stored packed. */
msa_status_t msa_gather_pages(const msa_varlen_t* seqs, const int32_t* block_table, int32_t max_blocks,
                              int64_t num_pages, int64_t row_bytes, const void* pages, void* packed, void* ws,
                              size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* Main Branch backward: the gradients of the attention over the support J
 * (the selected blocks' tokens cut at the query, or with dense != 0 every
 * token up to it) for an upstream gradient dout.  MSA is trained end to end,
 * so the forward that yifor-blog "設計核心" item 2 and pnsm.cn sec. 2 define
 * is differentiated like any softmax attention.  With P_j = exp(sm_scale
 * q_h.k_j - lse[t, h]), dP_j = dout_h.v_j, D = dout_h.out_h, dS_j = P_j (dP_j
 * - D):
 *   dq[t, h]  = sm_scale sum_j dS_j k_j                 (out, float [T, H, d])
 *   dk[j, g] += sm_scale dS_j q[t, h],  dv[j, g] += P_j dout[t, h]
 *                                                      (out, float [S, G, d];
 *               zeroed by the call, then accumulated atomically, so their
 *               rounding order varies from run to run)
 * out and lse are the forward's outputs for the same support (prefill or
 * dense call).  The selection is not differentiated.  ws:
 * msa_sparse_attn_backward_workspace_size bytes, 256-byte aligned.  A
 * selected block id past the query's block is recorded as
 * MSA_ERR_DEVICE_CHECK and left out.  k, v, dk and dv must be 16-byte
 * aligned (their rows are read and added 16 bytes at a time), and with
 * dense = 0 q, out, dout and dq too, else MSA_ERR_INVALID_ARG; d must be 64
 * or 128.  The selected support (dense = 0) runs on the tensor cores: the
 * selection is inverted into the forward's KV-outer lists; per work item the
 * key and value blocks stay in shared memory while the item's queries pass
 * in tiles of 128 (query, head) rows: S^T = K Q^T and dP^T = V dO^T, then
 * dV += P^T dO and dK += dS^T Q with P^T and dS^T in TMEM, and dQ = dS K;
 * dq is added per tile and dk / dv per item with vector reductions (dq's
 * rounding order varies from run to run too); P and dS enter the products
 * in bf16.  The dense support runs on the CUDA cores (one CTA per (query,
 * group), key and value rows staged per 64-token chunk). */
size_t msa_sparse_attn_backward_workspace_size(const msa_shape_t* shape, const msa_varlen_t* seqs, int32_t dense);

msa_status_t msa_sparse_attn_backward(const msa_shape_t* shape, const msa_varlen_t* seqs,
                                      const void* q,      /* device bf16 [T, H, d] */
                                      const void* k,      /* device bf16 [S, G, d] */
                                      const void* v,      /* device bf16 [S, G, d] */
                                      const int32_t* sel, /* device int32 [T, G, k]; NULL allowed when dense */
                                      const void* out,    /* device bf16 [T, H, d] */
                                      const float* lse,   /* device float [T, H] */
                                      const void* dout,   /* device bf16 [T, H, d] */
                                      int32_t dense, float* dq, float* dk, float* dv, void* ws, size_t ws_bytes,
                                      void* stream);

/* ---------------------------------------------------------------------- */
/* The FLOP-matched sliding-window baseline's selection (pnsm.cn sec. 6
 * "Learnable sink 和滑动窗口消融"; yhxrc.cn sec. 三): for every (query, group)
 * the first n_sink blocks and the k - n_sink most recent ones (the query's own
 * block last), ascending, -1 padded; every causal block when there are at most
 * k.  No index scores: sel has msa_index_topk's layout, so the main-branch
 * calls run the baseline unchanged.  0 <= n_sink < k.  ws: at least 256
 * bytes, 256-byte aligned (the error word). */
msa_status_t msa_select_window(const msa_shape_t* shape, const msa_varlen_t* seqs, int32_t n_sink,
                               int32_t* sel, /* device int32 [T, G, k] (out) */
                               void* ws, size_t ws_bytes, void* stream);

/* The Index Branch under the scored selection policies the pages compare the
 * final rule with (pnsm.cn sec. 3 and its forced sink / local ablation;
 * yhxrc.cn sec. 二): blocks 0 .. n_sink-1 and the n_local most recent ones
 * (the query's own included) are forced, the rest of the k by block score
 * (score desc, id asc; NaN as -inf); every causal block when there are at
 * most k.  n_sink = 0, n_local = 1 is msa_index_topk's rule.  Requires
 * n_sink >= 0, n_local >= 1, n_sink + n_local <= k, max_k_len <= 1M tokens.
 * sel as msa_index_topk; ws: at least 256 bytes, 256-byte aligned; k_idx
 * 16-byte aligned (its rows are read 16 bytes at a time), else
 * MSA_ERR_INVALID_ARG.  A CUDA-core form (one CTA per (query, group)). */
msa_status_t msa_index_topk_policy(const msa_shape_t* shape, const msa_varlen_t* seqs, int32_t n_sink,
                                   int32_t n_local, const void* q_idx, const void* k_idx, int32_t* sel, void* ws,
                                   size_t ws_bytes, void* stream);

/* The share of each head's dense causal attention weight that the selected
 * tokens hold, the monitor the pages report for the selection (yhxrc.cn sec.
 * 二): share[i] = exp(lse_sel[i] - lse_all[i]), with lse_sel from
 * msa_sparse_attn_prefill and lse_all from msa_dense_attn on the same layer
 * (both device float [T, H]; n = T * H). */
msa_status_t msa_selected_share(const float* lse_sel, const float* lse_all, int64_t n, float* share,
                                void* stream);

/* ---------------------------------------------------------------------- */
/* Index-alignment target (pnsm.cn sec. 4 "KL alignment", sec. 5 "Indexer
 * warmup"; yhxrc.cn sec. 二): for every query t and group g, the KL divergence
 * KL(P || Q) over the support J (the tokens of the selected blocks sel[t, g]
 * cut at the query, or with dense != 0 every token up to the query), where
 *   P_j = mean over the group's heads h of exp(sm_scale q_h.k_j - lse[t, h])
 *         (the Main Branch's attention on J: lse must be the log-sum-exp over
 *         the same J, as msa_sparse_attn_prefill returns it for the sparse
 *         support and msa_dense_attn for the dense one),
 *   Q_j = softmax over J of tau * <q_idx[t, g], k_idx[j]>  (the Index Branch).
 *   kl     device float [T, G] (out)
 *   lse_z  device float [T, G] (out, or NULL): the student's log-sum-exp
 *          log sum_j exp(z_j), which the backward call takes
 * The teacher P is a constant of this value (its gradient is not the index
 * branch's to follow).  ws: msa_index_kl_workspace_size bytes, 256-byte
 * aligned (the error word first).  A selected block id past the query's
 * block is recorded as MSA_ERR_DEVICE_CHECK and skipped.  k and k_idx must be 16-byte aligned
 * (their rows are read 16 bytes at a time), and with dense = 0 q_idx too,
 * else MSA_ERR_INVALID_ARG.
 * The selected support (dense = 0) runs on the tensor cores: the selection is
 * inverted into the forward's KV-outer lists, each selected block's keys and
 * index keys are loaded once per work item, S = Q K^T of its gathered queries
 * and their index scores Z = Q_idx K_idx^T are tcgen05 products, and the sums
 * are merged per (query, group); ws must then hold
 * msa_index_kl_workspace_size bytes (the lists and one 16-byte partial per
 * (query, group, slot)).  The dense support (the warm-up) runs on the CUDA
 * cores (one CTA per (query, group)) with the 256-byte workspace. */
size_t msa_index_kl_workspace_size(const msa_shape_t* shape, const msa_varlen_t* seqs, int32_t dense);

msa_status_t msa_index_kl(const msa_shape_t* shape, const msa_varlen_t* seqs,
                          const void* q,      /* device bf16 [T, H, d] */
                          const void* k,      /* device bf16 [S, G, d] */
                          const void* q_idx,  /* device bf16 [T, G, d_idx] */
                          const void* k_idx,  /* device bf16 [S, d_idx] */
                          const int32_t* sel, /* device int32 [T, G, k]; NULL allowed when dense */
                          const float* lse,   /* device float [T, H] */
                          float tau, int32_t dense, float* kl, float* lse_z, void* ws, size_t ws_bytes,
                          void* stream);

/* Gradient of sum_{t,g} KL(P || Q) with respect to the index query and the
 * index keys, the teacher held constant (pnsm.cn sec. 4 "gradient detach"):
 * with w_j = tau (Q_j - P_j) over the support of (t, g),
 *   dq_idx[t, g, :] = sum_j w_j k_idx[j, :]             (out, float [T, G, d_idx])
 *   dk_idx[j, :]    = sum over (t, g) of w_j q_idx[t, g, :]  (out, float [S, d_idx];
 *                     zeroed by the call, then accumulated atomically, so
 *                     its rounding order varies from run to run)
 * Arguments as msa_index_kl, plus lse_z from it; dk_idx must be 16-byte
 * aligned too (its rows are added 16 bytes at a time), and with dense = 0
 * dq_idx too.  The selected support (dense = 0) runs over the same plan and
 * workspace as msa_index_kl (msa_index_kl_workspace_size bytes): per work
 * item S and the index scores are tcgen05 products, w_j = tau (Q_j - P_j) per
 * (query, key) is formed from them, and both gradients are added with vector
 * reductions (their rounding order varies between runs); the dense support
 * runs on the CUDA cores with the 256-byte workspace. */
msa_status_t msa_index_kl_backward(const msa_shape_t* shape, const msa_varlen_t* seqs, const void* q,
                                   const void* k, const void* q_idx, const void* k_idx, const int32_t* sel,
                                   const float* lse, const float* lse_z, float tau, int32_t dense, float* dq_idx,
                                   float* dk_idx, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* Two-phase combine on its own (pnsm.cn sec. 7 "two-phase combine").
 * Merges, for every query t and head h = g*(H/G) + i of group g, the partials
 * of the slots s with sel[t, g, s] >= 0:
 *   part_acc  device f16 [T, G, k, d/8, H/G, 8]  softmax output over one block,
 *             normalised by its own sum: element (t, g, s, column 8c+e) of
 *             head i is at [t][g][s][c][i][e]
 *   part_lse  device f32 [T, G, k, H/G]          that block's log-sum-exp
 * into out[t, h, :] = sum_s exp(lse_s - LSE) * acc_s with LSE = log sum_s
 * exp(lse_s), and lse[t, h] = LSE (lse may be NULL).  part_acc and part_lse
 * must start on 16-byte boundaries (MSA_ERR_INVALID_ARG otherwise); every
 * query needs at least one slot with sel >= 0.  Slots with sel < 0 are never
 * read. */
msa_status_t msa_combine(const msa_shape_t* shape, int64_t T,
                         const void* part_acc, const float* part_lse, const int32_t* sel,
                         void* out, float* lse, void* stream);

/* ---------------------------------------------------------------------- */
/* Dense causal GQA attention (every key <= the query position), the
 * denominator of the pages' speedup comparison against GQA (pnsm.cn sec. 9).
 * Same layouts and argument rules as msa_sparse_attn_prefill without `sel`
 * (shape->k and shape->d_idx are ignored apart from the shape checks); the
 * workspace (msa_dense_attn_workspace_size bytes, 256-byte aligned) holds the
 * error word and the per-sequence tile counts.  A sequence with more queries
 * than keys records MSA_ERR_DEVICE_CHECK in the error word and gets no output.
 * Asynchronous on `stream`. */
size_t msa_dense_attn_workspace_size(const msa_shape_t* shape, const msa_varlen_t* seqs);

msa_status_t msa_dense_attn(const msa_shape_t* shape, const msa_varlen_t* seqs,
                            const void* q, const void* k, const void* v,
                            void* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* Work split of the prefill main branch (process-wide; returns the previous
 * value).  This library's own scheduling choice: the pages' kernel runs
 * KV-outer throughout (pnsm.cn sec. 7; yololab.net "KV Outer Gather Q").
 * The prefill call groups query rows into tiles of 2 x 128/max(H/G, 8)
 * consecutive queries of one sequence; a block chosen by at least `theta` of a
 * tile's queries (for one group) is attended query-tile-major, merged with an
 * online softmax into one result per query, instead of one KV-outer partial
 * per (query, block).  The selected token sets and the exact softmax are the
 * same either way; only the rounding order differs.
 *   theta < 0   automatic: ceil(5/8 x tile queries) (the default)
 *   theta == 0  off: every selection goes through the KV-outer lists
 *   theta >= 1  that threshold (1: every selected block of a tile)
 * Decode calls (one query per sequence) never use query tiles.  The value is
 * one atomic word: safe to set from any thread; a call reads it once, when
 * it starts, and uses that value throughout. */
int32_t msa_set_tile_threshold(int32_t theta);

/* Planning window of the prefill main branch's KV-outer lists (process-wide;
 * returns the previous value).  Also this library's scheduling choice: the
 * pages invert the selection into one query list per selected KV block
 * (pnsm.cn sec. 9 "reverse index"); here the lists are cut into windows of
 * `rows` consecutive query rows of a pass and keyed (group, window, block), so
 * the work items run group by group and, within a group, window by window:
 * the gathered query rows of the current window stay in L2, at the price of
 * loading a block once per window that selects it.  Results do not depend on
 * the value (each selection is attended exactly once either way).
 *   rows <= 0   the default (8192)
 *   otherwise   clamped to [128, 2^20]
 * The workspace size of msa_sparse_attn_prefill depends on it: query the size
 * after setting it.  One atomic word, read once per call. */
int32_t msa_set_attn_window(int32_t rows);

/* ---------------------------------------------------------------------- */
/* Decode of one long sequence split across ranks by key range (this
 * library's multi-GPU form of the pages' decode step, pnsm.cn sec. 9; the
 * pages select per query the top-k blocks of the whole cache with the local
 * block forced, sec. 2).  Rank r holds the keys [a_r, b_r) of each sequence
 * (block aligned, the last rank holding the query's local block); the query
 * is on every rank.  The global top-(k-1) is within the union of each range's
 * own top-(k-1), so:
 *   1. msa_index_topk_decode_candidates on each rank's key slice: per (query,
 *      group) the k-1 best blocks of the slice and their raw scores, in the
 *      selection order (score descending, lower id first), ids local to the
 *      slice; -1 / -inf padding.  all_blocks = 1 when the query lies after
 *      the slice's keys (every complete block is a candidate), 0 for the
 *      slice that ends with the query (its last block is the local block and
 *      is not scored, as in msa_index_topk).  Same workspace and checks as
 *      msa_index_topk's decode shape; k = 1 writes nothing.
 *      cand_ids int32 [T, G, k-1] and cand_scores f32 [T, G, k-1] (device).
 *   2. the callers exchange the candidates (ids made global by adding each
 *      slice's first block) and msa_merge_candidates merges n_cand of them
 *      per (query, group) under the same order, with local_block[b] (global
 *      id, device int32 [batch]) forced: sel int32 [batch, G, k] as
 *      msa_index_topk writes it.  A candidate id >= the local block is
 *      recorded as MSA_ERR_DEVICE_CHECK (site 181) and skipped; n_cand <= 256.
 *      ws: at least 256 bytes (the error word).
 *   3. msa_select_block_range cuts one rank's part out of a selection: ids in
 *      [blk_lo[b], blk_hi[b]) minus blk_lo[b], ascending, -1 padded (device
 *      int32 [batch] bounds; sel and sel_out [batch, G, k]); the rank then
 *      runs msa_sparse_attn_decode on its slice with it.
 *   4. the per-rank outputs are merged with msa_combine (one slot per rank).
 * All device buffers belong to the caller; errors before any launch as for
 * the other calls. */
msa_status_t msa_index_topk_decode_candidates(const msa_shape_t* shape, const msa_varlen_t* seqs,
                                              const void* q_idx, const void* k_idx, int32_t all_blocks,
                                              int32_t* cand_ids, float* cand_scores, void* ws, size_t ws_bytes,
                                              void* stream);
msa_status_t msa_merge_candidates(const msa_shape_t* shape, int32_t batch, int32_t n_cand,
                                  const int32_t* cand_ids, const float* cand_scores, const int32_t* local_block,
                                  int32_t* sel, void* ws, size_t ws_bytes, void* stream);
msa_status_t msa_select_block_range(const msa_shape_t* shape, int32_t batch, const int32_t* sel,
                                    const int32_t* blk_lo, const int32_t* blk_hi, int32_t* sel_out, void* stream);

/* ---------------------------------------------------------------------- */
/* Self-test of the bounded waits (no counterpart on the pages: a failure-
 * detection check of this library).  Every spin-wait in the kernels gives up
 * after about a second and records MSA_ERR_TIMEOUT in the call's error word
 * instead of hanging the GPU.  This call launches one small kernel whose two
 * waits can never end (an mbarrier nobody arrives on, a workspace counter
 * nobody advances), each with the library's own wait given `limit_us`
 * microseconds (1 ... 1,000,000); both give up, the kernel returns, and
 * msa_get_device_error(ws) then reads MSA_ERR_TIMEOUT (site 221).  The word
 * at ws + 256 + 4 (int32) counts the waits that ran out (2).
 * ws: device, 256-byte aligned, msa_selftest_wait_timeout_workspace_size()
 * bytes; cleared by the call.  Returns MSA_ERR_INVALID_ARG for a limit out of
 * range, MSA_ERR_WORKSPACE for a missing or short workspace, before any launch. */
size_t msa_selftest_wait_timeout_workspace_size(void);
msa_status_t msa_selftest_wait_timeout(uint32_t limit_us, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* Decode-shaped index top-k that allocates nothing (the pages have no
 * counterpart: this is a deployment convenience).
 *
 * For callers that cannot allocate device memory when they call in, such as a
 * serving loop whose framework reserves all device memory up front and hands
 * out no scratch buffers, or a host that forbids cudaMalloc on the decode path
 * because cudaMalloc synchronizes the device.  Same operation and layouts as
 * msa_index_topk with max_q_len <= 1 (one query per sequence); the caller still
 * passes the inputs and `sel`.  Arguments are checked as msa_index_topk checks
 * them, in the same order; with no queries the data pointers may be NULL.
 *
 * Scratch: a fixed array inside the library, msa_index_topk_decode_noalloc_
 * max_scratch() bytes (16 MiB) per GPU, held by every GPU that loads the
 * library until the process exits.  The need is 4*G bytes per cached block
 * plus small offsets, so the array holds about 1.05 million blocks: about
 * 134 million cached tokens (sum of the cache lengths) at G = 4 and B_k = 128.
 * A call whose scratch need (msa_index_topk_workspace_size) exceeds it returns
 * MSA_ERR_WORKSPACE and launches nothing.  Calls and allocations: none (no
 * cudaMalloc/cudaFree).
 * The first call on a device looks the array's device address up (with that
 * device current) and keeps it; make that first call before any stream capture.
 * A cudaDeviceReset of that device ends the use of this entry point on it for
 * the rest of the process (the kept address would be stale).
 * All calls on one device share its array, which keeps the last call's
 * contents (each call clears the error word it needs zeroed): calls that
 * overlap on the same device (different streams) race, so order them; calls
 * on different devices use separate copies.
 * device_error (device int32, may be NULL) receives the call's device error
 * code (an msa_status_t, MSA_OK if none), stream-ordered after the call. */
size_t msa_index_topk_decode_noalloc_max_scratch(void);

msa_status_t msa_index_topk_decode_noalloc(const msa_shape_t* shape, const msa_varlen_t* seqs,
                                           const void* q_idx,   /* device bf16 [T, G, d_idx] */
                                           const void* k_idx,   /* device bf16 [S, d_idx] */
                                           int32_t* sel,        /* device int32 [T, G, k] (out) */
                                           int32_t* device_error, /* device int32 [1] (out) or NULL */
                                           void* stream);

/* ---------------------------------------------------------------------- */
/* Measurement support (for benchmarks; no counterpart in the method).
 * msa_profile_enable(1) makes every kernel launch of the library record a CUDA
 * event pair on its launch stream; msa_profile_read(name, ...) waits for those
 * events and returns the summed device time (ms) and launch count of the
 * kernel `name` ("index_topk_prefill", "decode_scan", "decode_select",
 * "sparse_attn", "combine", "count", "plan", "scatter", "dense_attn", ...).
 * With name == NULL it returns the number of kernels launched since the last
 * msa_profile_reset (launches are counted even while timing is disabled). */
msa_status_t msa_profile_enable(int on);
msa_status_t msa_profile_reset(void);
msa_status_t msa_profile_read(const char* kernel, double* total_ms, int64_t* count);

/* ---------------------------------------------------------------------- */
/* Device error word of a workspace.  Waits for `stream`, copies the word to
 * the host and clears it.  *code is an msa_status_t (MSA_OK if none);
 * *where names the kernel site, *info0 / *info1 carry details.  The first
 * failure of a call is kept.  Sites (where):
 *   101-104  prefill index top-k (loads, MMA, epilogue, a sequence with T_b > S_b;
 *            info0 = sequence, info1 = T_b for 104)
 *   111      decode index scan / selection (info0 = sequence)
 *   121      a selection row with an id past the query's block, or not ids-first
 *            (info0 = query row, info1 = block id)
 *   131-134  KV-outer attention (loads, MMA, softmax, work items)
 *   141      dense attention (info0 = sequence with T_b > S_b)
 *   151-154  query-tile attention (scheduler, loads, MMA, softmax)
 *   161      paged decode: a page outside the cache or a bad length
 *   171      index-alignment target / its gradient   181  window selection
 *   191      main-branch backward                      201  policy selection
 *   211      page gather (info0 = sequence, info1 = block)
 *   221      bounded-wait self-test              231  decode candidate merge
 * MSA_ERR_TIMEOUT codes come from a bounded wait that ran out (about a
 * second); the call's results are then not valid, the context still is. */
msa_status_t msa_get_device_error(void* ws, int32_t* code, int32_t* where, int32_t* info0,
                                  int32_t* info1, void* stream);

/* Library version string. */
const char* msa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */
