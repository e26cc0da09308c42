"""Plain fp64 CPU oracle of the selection-policy variants that the MSA pages
compare the final rule with: forced sink blocks, a forced local window, the
FLOP-matched sliding-window baseline, and other block sizes.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this module: only the tests may use it.  It shares no code with the CUDA path.
No kernel implements these variants yet (the kernels keep the final rule:
the local block forced, B_k = 128); this oracle comes first, pinned.

Sources (web pages about MSA; cited by title / address and section):

* [pnsm]  "MiniMax Sparse Attention：一篇读懂百万上下文时代的稀疏注意力工程化路线"
  (pnsm.cn), sec. 3 "Attention sink：为什么第一个 token 仍然重要" (the trained
  selector picks the first block by itself; the forced sink / local ablation
  of the appendix changes little, and only the local block stays forced),
  sec. 6 "Learnable sink 和滑动窗口消融" (a fixed first block + local window
  with the same token budget, the FLOP-matched sliding-window baseline), and
  its ablation table (block sizes 32 / 64 / 128; forced sink / local).
* [yhxrc] M3 / MSA comparison article (yhxrc.cn), sec. 二 "MSA是怎么做的"
  (early versions forced the first block and a nearby local window; the
  final rule forces only the current block) and sec. 三 (the FLOP-matched
  baseline: the first block plus the most recent window, same budget).

The general rule written here (a reading: the pages name the variants, not a
formula):

    forced(lb) = {0 .. n_sink-1} ∪ {lb-n_local+1 .. lb}, cut to blocks 0..lb;
    sel = all causal blocks 0..lb            if lb + 1 <= k,
          forced ∪ best (k - |forced|) of the other causal blocks by
          (block score descending, block index ascending)   otherwise.

* the final MSA rule is n_sink = 0, n_local = 1 (only the local block);
* the early forced sink / local variant is n_sink >= 1 with n_local >= 1;
* the FLOP-matched sliding-window baseline is n_sink = 1, n_local = k - 1:
  nothing is left to the scores, every query keeps k blocks;
* other block sizes: B_k is a parameter (the block max-pool and the causal
  cut follow it);
* n_sink + n_local <= k is required (ValueError otherwise).
"""
from __future__ import annotations

from typing import List, Sequence

import numpy as np

from oracle import msa_oracle as O

__all__ = ["forced_blocks", "select_blocks_policy", "index_topk_policy", "window_baseline"]


def forced_blocks(lb: int, n_sink: int, n_local: int) -> List[int]:
    """Blocks a query in local block lb keeps regardless of scores."""
    f = set(range(min(n_sink, lb + 1)))
    f |= set(range(max(0, lb - n_local + 1), lb + 1))
    return sorted(f)


def select_blocks_policy(S, k: int, n_sink: int = 0, n_local: int = 1) -> List[int]:
    """S holds the block scores of blocks 0..lb (lb the query's own block).
    Returns the selected blocks, ascending (see the module comment)."""
    if n_sink < 0 or n_local < 1 or n_sink + n_local > k:
        raise ValueError("need n_sink >= 0, n_local >= 1 and n_sink + n_local <= k")
    S = np.asarray(S, dtype=np.float64)
    lb = S.shape[0] - 1
    if lb < 0:
        return []
    if lb + 1 <= k:
        return list(range(lb + 1))
    forced = forced_blocks(lb, n_sink, n_local)
    fset = set(forced)
    cand = np.array([b for b in range(lb + 1) if b not in fset], dtype=np.int64)
    keys = S[cand]
    keys = np.where(np.isnan(keys), -np.inf, keys)
    order = np.lexsort((cand, -keys))          # score descending, then index ascending
    chosen = [int(cand[i]) for i in order[: k - len(forced)]]
    return sorted(fset | set(chosen))


def window_baseline(lb: int, k: int) -> List[int]:
    """The FLOP-matched sliding-window baseline written out: the first block
    and the k-1 most recent ones (all causal blocks when lb + 1 <= k)."""
    if lb + 1 <= k:
        return list(range(lb + 1))
    return [0] + list(range(lb - k + 2, lb + 1))


def index_topk_policy(q_idx, k_idx, cu_q: Sequence[int], cu_k: Sequence[int], k: int, B_k: int,
                      n_sink: int = 0, n_local: int = 1) -> np.ndarray:
    """Index branch under a selection policy: sel[t, g, :] ascending, -1 padded
    (scores and block max-pool as in the final rule, for any B_k)."""
    q_idx = np.asarray(q_idx, dtype=np.float64)
    k_idx = np.asarray(k_idx, dtype=np.float64)
    T, G, _ = q_idx.shape
    sel = np.full((T, G, k), -1, dtype=np.int32)
    for b in range(len(cu_q) - 1):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
        for i, pos in enumerate(O.query_positions(q1 - q0, k1 - k0)):
            for g in range(G):
                s = O.index_scores(q_idx[q0 + i, g], k_idx[k0:k1], int(pos))
                blocks = select_blocks_policy(O.block_max_pool(s, B_k), k, n_sink, n_local)
                sel[q0 + i, g, : len(blocks)] = blocks
    return sel
