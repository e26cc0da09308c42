"""Plain fp64 CPU oracle of the MiniMax Sparse Attention (MSA) forward pass.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may use it.  It shares no code with the CUDA path; the two
meet only in the seeded input generators, which hold none of the method's
arithmetic.

Sources (web pages about MSA; cited by title / address and section):

* [pnsm]  "MiniMax Sparse Attention：一篇读懂百万上下文时代的稀疏注意力工程化路线"
  (pnsm.cn), sec. 2 "MSA 的核心：在 GQA 上做 group-specific block selection",
  sec. 7 "Kernel 设计".
* [yifor] "MiniMax Sparse Attention (MSA): a Two-Branch Block-Sparse Attention
  Trained on a 109B-Parameter MoE With a 3T-Token Budget" (yifor-blog), sections
  "設計核心：將注意力拆分為「索引」與「主路徑」兩路分支" and "從 O(N) 降至 O(kB_k)".
* [yhxrc] M3 / MSA comparison article (yhxrc.cn), sec. 二 "MSA是怎么做的".
* [yololab] MiniMax M3 article (yololab.net), "MSA的兩個主要步驟".

What the pages fix, and what this module does step by step:

1. Index score ([pnsm] sec. 7 "exp-free Top-k"; [yhxrc] sec. 二): one index
   query head per GQA group is dotted with one index key head shared by all
   groups; the raw dot product is the token score, no softmax and no exp,
   because softmax keeps the order of scores.
2. Block max-pooling ([yifor] "設計核心" item 1; [yhxrc] sec. 二 "block max
   pooling"): the score of a 128-token block is the largest token score in it.
3. Top-k with the forced local block ([pnsm] sec. 2 third point; [yhxrc]
   sec. 二: "the block holding the current position is always chosen, the rest by
   score"): k counts the local block, so k-1 blocks are chosen by score.
4. Main branch ([yifor] "設計核心" item 2; [yololab] step 2): exact softmax
   attention of every query head of the group over the tokens of the selected
   blocks, causal (tokens after the query are not visible).

Readings where the pages are silent (each one is listed in the design notes):

* ties at the k-th place go to the lower block index;
* NaN token scores rank as -inf; blocks whose score is -inf still fill free
  slots in ascending index order, so a query always gets min(k, nb) blocks;
* when a query has nb <= k causal blocks, all of them are selected;
* the main-branch softmax scale ``sm_scale`` is an argument (1/sqrt(d) by
  default); the index score has no scale;
* group g serves query heads [g*H/G, (g+1)*H/G) (the usual GQA map);
* the queries of sequence b are its last T_b tokens: query i sits at absolute
  position S_b - T_b + i (prefill: T_b = S_b; decode: T_b = 1, the new token at
  position L-1, with the cache already holding it);
* ``lse`` is the natural-log log-sum-exp of the scaled scores over the
  selected token set.

Parity status: every function below is pinned by a CPU test against something
other than itself (brute force, a closed form, an identity or a library
routine); see ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

import numpy as np

__all__ = [
    "query_positions",
    "index_scores",
    "block_max_pool",
    "select_blocks",
    "index_topk",
    "index_topk_rows",
    "attend",
    "selected_token_set",
    "main_branch",
    "msa_forward_rows",
    "lse_combine",
    "invert_selection",
    "block_candidates",
    "merge_block_candidates",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def query_positions(T_b: int, S_b: int) -> np.ndarray:
    """Absolute positions of the T_b queries of a sequence with S_b keys: the
    queries are the last T_b tokens (reading for prefill, decode and chunks)."""
    if T_b > S_b:
        raise ValueError("a sequence cannot have more queries than keys")
    return np.arange(S_b - T_b, S_b, dtype=np.int64)


def index_scores(q_idx_tg, k_idx_seq, pos: int) -> np.ndarray:
    """Step 1.  s_j = <q_idx[t,g], k_idx[j]> for every causal key j in [0, pos].

    Plain dot products in fp64, no scale, no exp ([pnsm] sec. 7 exp-free Top-k;
    [yhxrc] sec. 二: scoring skips the exponential since only the ranking
    matters)."""
    q = _f64(q_idx_tg)
    kk = _f64(k_idx_seq)[: pos + 1]
    return kk @ q


def block_max_pool(s, B_k: int) -> np.ndarray:
    """Step 2.  S_b = max_{j in block b} s_j over the tokens of s (the last block
    may be partial).  NaN scores count as -inf ([yifor] "Max-pooling";
    [yhxrc] sec. 二 "block max pooling")."""
    s = _f64(s)
    n = s.shape[0]
    nb = -(-n // B_k)
    padded = np.full(nb * B_k, -np.inf)
    padded[:n] = np.where(np.isnan(s), -np.inf, s)
    return padded.reshape(nb, B_k).max(axis=1)


def select_blocks(S, k: int) -> List[int]:
    """Step 3.  S holds the block scores of blocks 0..lb, lb being the query's own
    (local) block.  The local block is always selected; the other k-1 are the
    best of blocks 0..lb-1 in the order (score descending, index ascending).
    With lb+1 <= k every causal block is selected.  Returned ascending.

    ([pnsm] sec. 2 "local block 始终保留" and the 16 x 128 = 2048 budget;
    [yhxrc] sec. 二: the block of the current position is mandatory, the rest by
    score, 16 blocks in total.)"""
    S = _f64(S)
    lb = S.shape[0] - 1
    if lb < 0:
        return []
    if lb + 1 <= k:
        return list(range(lb + 1))
    cand = np.arange(lb)
    keys = np.where(np.isnan(S[:lb]), -np.inf, S[:lb])
    # lexsort sorts by the last key first: score descending, then index ascending
    order = np.lexsort((cand, -keys))
    chosen = sorted(int(b) for b in order[: k - 1])
    return chosen + [lb]


def index_topk_rows(q_idx_rows, k_idx_seq, positions: Sequence[int], k: int, B_k: int,
                    row_chunk: int = 16) -> np.ndarray:
    """Steps 1-3 for some queries of ONE sequence: sel[r, g, :] for the query at
    absolute position positions[r] (ascending ids, -1 padded).

    The token scores of a few rows at a time come from one matrix product
    (k_idx[0..p_max] times their index queries); each row then keeps only its
    causal keys j <= p, exactly as in ``index_scores``."""
    q = _f64(q_idx_rows)
    R, G, _ = q.shape
    sel = np.full((R, G, k), -1, dtype=np.int32)
    for r0 in range(0, R, row_chunk):
        r1 = min(R, r0 + row_chunk)
        pmax = int(max(positions[r0:r1]))
        kk = _f64(k_idx_seq[: pmax + 1])
        s_all = kk @ q[r0:r1].reshape((r1 - r0) * G, -1).T   # [pmax+1, rows*G]
        for r in range(r0, r1):
            p = int(positions[r])
            for g in range(G):
                s = s_all[: p + 1, (r - r0) * G + g]
                blocks = select_blocks(block_max_pool(s, B_k), k)
                sel[r, g, : len(blocks)] = blocks
    return sel


def index_topk(q_idx, k_idx, cu_q: Sequence[int], cu_k: Sequence[int], k: int,
               B_k: int) -> np.ndarray:
    """Index branch end to end: sel[t, g, :] = ascending selected block ids of
    query t for group g (ids local to t's sequence), padded with -1.

    q_idx: [T, G, d_idx]; k_idx: [S, d_idx] (packed sequences, offsets cu_q and
    cu_k)."""
    q_idx = np.asarray(q_idx)
    T, G, _ = q_idx.shape
    sel = np.full((T, G, k), -1, dtype=np.int32)
    for b in range(len(cu_q) - 1):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
        if q1 == q0:
            continue
        pos = query_positions(q1 - q0, k1 - k0)
        sel[q0:q1] = index_topk_rows(q_idx[q0:q1], np.asarray(k_idx)[k0:k1], pos, k, B_k)
    return sel


def selected_token_set(blocks: Sequence[int], pos: int, B_k: int) -> np.ndarray:
    """Tokens the main branch attends to: the union of the selected blocks,
    cut causally at the query position (only the local block can reach past it)."""
    parts = []
    for b in blocks:
        if b < 0:
            continue
        lo = b * B_k
        hi = min((b + 1) * B_k, pos + 1)
        if hi > lo:
            parts.append(np.arange(lo, hi, dtype=np.int64))
    if not parts:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate(parts)


def attend(q_tg, K_J, V_J, sm_scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Exact softmax attention of the query heads q_tg [Hg, d] over the token set
    whose keys / values are K_J, V_J [|J|, d], in fp64.  Returns (o [Hg, d],
    lse [Hg]), lse the natural log-sum-exp of the scaled scores."""
    q = _f64(q_tg)
    Kj = _f64(K_J)
    Vj = _f64(V_J)
    s = sm_scale * (q @ Kj.T)                      # [Hg, |J|]
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    o = (e @ Vj) / l
    lse = (m + np.log(l))[:, 0]
    return o, lse


def main_branch(q_tg, K_g, V_g, blocks: Sequence[int], pos: int, B_k: int,
                sm_scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Step 4.  Exact softmax attention of the query heads of one group over the
    selected tokens ([yifor] "Main Branch"; [yololab] step 2 "精確注意力").

    q_tg: [Hg, d] query heads of the group; K_g, V_g: [S_b, d] the group's keys
    and values of this sequence.  Returns (o [Hg, d], lse [Hg])."""
    J = selected_token_set(blocks, pos, B_k)
    return attend(q_tg, np.asarray(K_g)[J], np.asarray(V_g)[J], sm_scale)


def msa_forward_rows(q, k, v, sel, cu_q, cu_k, rows: Sequence[int], B_k: int,
                     sm_scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Main branch for the listed query rows, given the selection sel[T, G, k].

    q: [T, H, d]; k, v: [S, G, d].  Returns (o [len(rows), H, d],
    lse [len(rows), H])."""
    T, H, d = q.shape
    G = k.shape[1]
    Hg = H // G
    cu_q = np.asarray(cu_q, dtype=np.int64)
    cu_k = np.asarray(cu_k, dtype=np.int64)
    out = np.zeros((len(rows), H, d))
    lse = np.zeros((len(rows), H))
    for r, t in enumerate(rows):
        b = int(np.searchsorted(cu_q, t, side="right") - 1)
        T_b = int(cu_q[b + 1] - cu_q[b])
        S_b = int(cu_k[b + 1] - cu_k[b])
        pos = S_b - T_b + (t - int(cu_q[b]))
        k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
        for g in range(G):
            o, ls = main_branch(q[t, g * Hg:(g + 1) * Hg], k[k0:k1, g], v[k0:k1, g],
                                [int(x) for x in sel[t, g]], pos, B_k, sm_scale)
            out[r, g * Hg:(g + 1) * Hg] = o
            lse[r, g * Hg:(g + 1) * Hg] = ls
    return out, lse


def lse_combine(accs, lses) -> Tuple[np.ndarray, np.ndarray]:
    """Two-phase combine ([pnsm] sec. 7 "two-phase combine"): merge softmax
    partials over disjoint token sets.  accs[i] is the normalised output over set
    i and lses[i] its log-sum-exp; the result is the softmax output over the
    union: LSE = log sum_i exp(lse_i), o = sum_i exp(lse_i - LSE) acc_i."""
    accs = _f64(accs)
    lses = _f64(lses)
    m = np.max(lses, axis=0)
    w = np.exp(lses - m)
    tot = w.sum(axis=0)
    LSE = m + np.log(tot)
    o = np.einsum("i...,i...d->...d", w / tot, accs)
    return o, LSE


def invert_selection(sel, cu_q, cu_k, B_k: int) -> Dict[Tuple[int, int, int], List[int]]:
    """Reverse index ([pnsm] sec. 9 lists "反向索引" among the kernel costs;
    KV-outer gathers, per KV block, the queries that chose it).

    Returns {(sequence, group, block): ascending list of query rows t that
    selected that block}."""
    sel = np.asarray(sel)
    T, G, k = sel.shape
    cu_q = np.asarray(cu_q, dtype=np.int64)
    lists: Dict[Tuple[int, int, int], List[int]] = {}
    for b in range(len(cu_q) - 1):
        for t in range(int(cu_q[b]), int(cu_q[b + 1])):
            for g in range(G):
                for blk in sel[t, g]:
                    if blk < 0:
                        continue
                    lists.setdefault((b, g, int(blk)), []).append(t)
    return lists


# --------------------------------------------- key-range split of a decode ---
#
# Step 3 over a cache cut into key ranges: the k-1 blocks a query chooses by
# score are the first k-1 of all its non-local blocks under the order (score
# descending, index ascending), so they are also the first k-1 of the union of
# every range's own first k-1.  These two functions restate step 3 in that
# form; with the whole cache as one range they reduce to ``select_blocks``.


def block_candidates(S, k: int) -> Tuple[List[int], List[float]]:
    """The first k-1 blocks of one key range under the order of step 3 (score
    descending, index ascending; NaN as -inf), with their scores.  S holds the
    scores of the range's competing blocks (none of them the query's local
    block), indexed from 0."""
    S = _f64(S)
    keys = np.where(np.isnan(S), -np.inf, S)
    order = np.lexsort((np.arange(keys.shape[0]), -keys))[: max(k - 1, 0)]
    return [int(b) for b in order], [float(keys[b]) for b in order]


def merge_block_candidates(ids: Sequence[int], scores: Sequence[float], lb: int, k: int) -> List[int]:
    """Step 3 from the candidates of several ranges (global block ids, all
    below the local block lb): the first k-1 of them under the same order,
    then the local block; returned ascending."""
    ids = np.asarray(list(ids), dtype=np.int64)
    keys = np.asarray(list(scores), dtype=np.float64)
    keys = np.where(np.isnan(keys), -np.inf, keys)
    order = np.lexsort((ids, -keys))[: max(k - 1, 0)]
    return sorted(int(ids[o]) for o in order) + [int(lb)]
