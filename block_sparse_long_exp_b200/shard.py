"""Splitting one long sequence's prefill across ranks by query ranges.

A query's result depends only on its own position and the keys before it, so
rank r can compute the queries [a_r, b_r) of a sequence by itself as a chunked
prefill: queries [a_r, b_r) over keys [0, b_r) (the calls take the queries of
a sequence as its last T_b tokens).  No collective is needed while the output
stays sharded; the keys [0, b_r) must be present on rank r.

The work per query grows with its position (the index branch scores every
earlier block), so equal row counts would leave the last rank the most work:
the ranges are cut at equal shares of the algorithmic work instead.

The backward of such a split has one exchange step.  Rank r's chunk reaches
the keys [0, b_r), so its dk, dv (and the index-alignment target's dk_idx)
hold only its own queries' contributions to those rows.  The layer's key-side
gradients are the sum of these over the ranks (sum_key_grads).  dq and dq_idx
stay sharded with the queries, as the output does.

A layer can also be split by GQA group (split_groups, group_slice): each rank
runs the whole path on its G / world groups and their query heads, with the
index keys replicated, and no collective unless the output is wanted whole
(gather_heads: one all-gather over the heads).
"""
from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

import numpy as np


def query_work(S: int, H: int, G: int, d: int, d_idx: int, B_k: int, k: int) -> np.ndarray:
    """Algorithmic FLOPs of each query position 0 .. S-1 of a prefill (index
    branch: 2 G d_idx B_k (nb - 1) when nb > k; main branch: 4 H d att)."""
    p = np.arange(S, dtype=np.int64)
    nb = p // B_k + 1
    idx = np.where(nb > k, 2 * G * d_idx * B_k * (nb - 1), 0)
    att = np.where(nb > k, (k - 1) * B_k + p % B_k + 1, p + 1)
    return (idx + 4 * H * d * att).astype(np.float64)


def split_query_ranges(work: np.ndarray, world: int, align: int = 1) -> List[Tuple[int, int]]:
    """Contiguous ranges [a, b) covering 0 .. len(work) whose work sums are as
    equal as cuts at multiples of `align` allow (a rank may get an empty range
    only when there are fewer aligned rows than ranks)."""
    n = len(work)
    if world < 1:
        raise ValueError("world must be >= 1")
    csum = np.concatenate([[0.0], np.cumsum(work)])
    cuts = [0]
    for r in range(1, world):
        target = csum[-1] * r / world
        c = int(np.searchsorted(csum, target))
        c = min(n, max(cuts[-1], int(round(c / align)) * align))
        cuts.append(c)
    cuts.append(n)
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


def chunk_of(inp: Dict[str, object], a: int, b: int) -> Dict[str, object]:
    """The inputs of one sequence's prefill (q/q_idx [S, ...], k/v/k_idx
    [S, ...], torch tensors) cut to the chunked call of queries [a, b): queries
    rows a .. b-1, keys rows 0 .. b-1, offsets [0, b-a] and [0, b]."""
    import torch
    dev = inp["q"].device
    return {
        "q": inp["q"][a:b], "q_idx": inp["q_idx"][a:b],
        "k": inp["k"][:b], "v": inp["v"][:b], "k_idx": inp["k_idx"][:b],
        "cu_q": torch.tensor([0, b - a], dtype=torch.int32, device=dev),
        "cu_k": torch.tensor([0, b], dtype=torch.int32, device=dev),
        "cu_q_host": [0, b - a], "cu_k_host": [0, b],
    }


def sum_key_grads(grads: Sequence[object], S: int, group=None) -> List[object]:
    """Key-side gradients of a query-range split summed over the ranks.

    grads: this rank's tensors [b_r, ...] (dk, dv, dk_idx: rows 0 .. b_r-1 of
    the sequence's keys, the rows its chunk reaches).  Each is placed in a zero
    tensor [S, ...]; all of them are summed across the process group by one
    all-reduce over a flat buffer (NCCL on the GPUs, gloo on the host); without
    an initialised group the padded tensors are returned as they are.  Returns
    the [S, ...] sums, equal on every rank."""
    import torch
    import torch.distributed as dist
    full = []
    for g in grads:
        if g.dim() < 1 or g.shape[0] > S:
            raise ValueError(f"a key-side gradient has {g.shape[0] if g.dim() else 0} rows, more than S = {S}")
        t = torch.zeros((S,) + tuple(g.shape[1:]), dtype=g.dtype, device=g.device)
        t[:g.shape[0]] = g
        full.append(t)
    if not (dist.is_available() and dist.is_initialized()) or not full:
        return full
    if len({(t.dtype, t.device) for t in full}) != 1:
        raise ValueError("the key-side gradients must share one dtype and device")
    flat = torch.cat([t.reshape(-1) for t in full])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    out, at = [], 0
    for t in full:
        out.append(flat[at:at + t.numel()].view(t.shape))
        at += t.numel()
    return out


def split_groups(G: int, world: int) -> List[Tuple[int, int]]:
    """GQA groups [g0, g1) of each rank for a group-sharded prefill: G / world
    consecutive groups each (world must divide G).  Every group's index
    branch and main branch are independent of the others'; only the index
    keys are shared, so they are replicated."""
    if world < 1 or G % world:
        raise ValueError(f"{world} ranks cannot share {G} groups evenly")
    n = G // world
    return [(r * n, (r + 1) * n) for r in range(world)]


def group_slice(inp: Dict[str, object], H: int, G: int, g0: int, g1: int) -> Dict[str, object]:
    """The inputs of groups [g0, g1) of a layer, as a layer of g1 - g0 groups:
    their query heads [g0 H/G, g1 H/G) of q, their rows of k, v and q_idx,
    and every index key.  The library's calls take it with the shape
    (H (g1 - g0) / G heads, g1 - g0 groups); the offsets are unchanged."""
    Hg = H // G
    out = dict(inp)
    out["q"] = inp["q"][:, g0 * Hg:g1 * Hg].contiguous()
    out["k"] = inp["k"][:, g0:g1].contiguous()
    out["v"] = inp["v"][:, g0:g1].contiguous()
    out["q_idx"] = inp["q_idx"][:, g0:g1].contiguous()
    return out


def gather_heads(out_part, group=None):
    """The full output [T, H, d] from every rank's heads [T, H / world, d] of
    a group-sharded prefill (one all-gather; ranks hold consecutive groups in
    rank order).  Without an initialised group the part is returned."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return out_part
    parts = [torch.empty_like(out_part) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, out_part.contiguous(), group=group)
    return torch.cat(parts, dim=1)


def imbalance(work: np.ndarray, ranges: List[Tuple[int, int]]) -> float:
    """Largest rank's work over the mean (1.0 = perfect balance)."""
    per = [float(work[a:b].sum()) for a, b in ranges]
    return max(per) / (sum(per) / len(per))


def decode_shards(lengths, world: int) -> List[List[int]]:
    """Decode sequences split across ranks: longest first, each to the rank
    with the least cached tokens so far (the decode step streams every cached
    index key, so its time follows the cached length).  Returns each rank's
    sequence ids, ascending."""
    if world < 1:
        raise ValueError("world must be >= 1")
    load = [0] * world
    out: List[List[int]] = [[] for _ in range(world)]
    for i in sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i)):
        r = min(range(world), key=lambda r: (load[r], r))
        out[r].append(i)
        load[r] += int(lengths[i])
    return [sorted(o) for o in out]


# ---------------------------------------------- decode split by key range ---
#
# One very long decode sequence can be cut by key range: rank r holds the
# keys of a consecutive run of blocks of every sequence (the last rank holds
# the block of the query), the query itself is on every rank.  The selection
# needs the top k-1 blocks of the whole cache; it is within the union of each
# range's own top k-1 (msa_index_topk_decode_candidates), exchanged with one
# small all-gather and merged by the library (msa_merge_candidates).  Each
# rank then attends its own selected blocks (msa_select_block_range +
# msa_sparse_attn_decode) and the per-rank outputs are merged by log-sum-exp
# (msa_combine, one slot per rank) after one more all-gather.


def split_key_blocks(L: int, world: int, B_k: int) -> List[Tuple[int, int]]:
    """Block ranges [lo, hi) of each rank for a cache of L tokens (blocks of
    B_k, the query at position L-1): the ceil(L / B_k) blocks cut into world
    consecutive runs as equal as possible; the last run holds the query's
    block.  Every rank needs at least one block."""
    nb = -(-int(L) // B_k)
    if world < 1 or nb < world:
        raise ValueError(f"{nb} blocks cannot be split over {world} ranks")
    cuts = [r * nb // world for r in range(world + 1)]
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


def key_slice(inp: Dict[str, object], lengths: Sequence[int], rank: int, world: int, B_k: int) -> Dict[str, object]:
    """Rank `rank`'s part of a decode batch (one query per sequence; k, v,
    k_idx packed over the sequences with offsets cu_k): every query and its
    q_idx, the keys of the rank's block range of each sequence, packed, and
    per sequence the range's first / last-plus-one block (blk_lo, blk_hi,
    global ids) and the query's local block.  all_blocks is True unless the
    rank holds the queries' blocks (the last rank): its keys then all lie
    before the query."""
    import torch
    dev = inp["q"].device
    cu = inp["cu_k_host"]
    rows, cu_k, lo, hi, local = [], [0], [], [], []
    for b, L in enumerate(lengths):
        a, z = split_key_blocks(L, world, B_k)[rank]
        k0, k1 = cu[b] + a * B_k, cu[b] + min(z * B_k, L)
        rows.append(torch.arange(k0, k1, device=dev))
        cu_k.append(cu_k[-1] + (k1 - k0))
        lo.append(a)
        hi.append(z)
        local.append((L - 1) // B_k)
    idx = torch.cat(rows)
    out = dict(inp)
    for name in ("k", "v", "k_idx"):
        out[name] = inp[name].index_select(0, idx).contiguous()
    i32 = lambda v: torch.tensor(v, dtype=torch.int32, device=dev)  # noqa: E731
    out.update(cu_k=i32(cu_k), cu_k_host=cu_k, blk_lo=i32(lo), blk_hi=i32(hi), local_block=i32(local),
               all_blocks=rank < world - 1)
    return out


def gather_candidates(ids, scores, blk_lo, group=None):
    """Every rank's candidates [B, G, c] (ids local to its range, -1 = none)
    made global (+ blk_lo[b]) and joined over the ranks along the last axis
    (one all-gather of ids and scores; without an initialised group the
    rank's own, made global)."""
    import torch
    import torch.distributed as dist
    glob = torch.where(ids >= 0, ids + blk_lo.view(-1, 1, 1).to(ids.dtype), ids)
    if not (dist.is_available() and dist.is_initialized()):
        return glob, scores
    n = dist.get_world_size(group)
    gi = [torch.empty_like(glob) for _ in range(n)]
    gs = [torch.empty_like(scores) for _ in range(n)]
    dist.all_gather(gi, glob.contiguous(), group=group)
    dist.all_gather(gs, scores.contiguous(), group=group)
    return torch.cat(gi, dim=2), torch.cat(gs, dim=2)


def rank_partials(outs, lses, sels, H: int, G: int):
    """The per-rank decode outputs laid out for msa_combine with one slot per
    rank: part_acc f16 [B, G, R, d/8, H/G, 8], part_lse f32 [B, G, R, H/G],
    slot sel int32 [B, G, R] (the rank's index where its range view of the
    selection, sels[r] [B, G, k], holds a block, else -1).  outs[r] bf16
    [B, H, d] and lses[r] f32 [B, H] are rank r's normalised output and
    log-sum-exp over its own selected tokens."""
    import torch
    R = len(outs)
    B, _, d = outs[0].shape
    Hg = H // G
    acc = torch.stack(outs).view(R, B, G, Hg, d // 8, 8).permute(1, 2, 0, 4, 3, 5).contiguous().half()
    lse = torch.stack(lses).view(R, B, G, Hg).permute(1, 2, 0, 3).contiguous()
    has = torch.stack([(s >= 0).any(dim=2) for s in sels])            # [R, B, G]
    rank_id = torch.arange(R, dtype=torch.int32, device=has.device).view(R, 1, 1).expand_as(has)
    slot = torch.where(has, rank_id, torch.full_like(rank_id, -1)).permute(1, 2, 0).contiguous()
    return acc, lse, slot


def gather_rank_outputs(out, lse, sel_local, group=None):
    """All ranks' outputs, log-sum-exps and range views (lists in rank order;
    one all-gather each; without an initialised group the rank's own)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return [out], [lse], [sel_local]
    n = dist.get_world_size(group)
    res = []
    for t in (out, lse, sel_local):
        parts = [torch.empty_like(t) for _ in range(n)]
        dist.all_gather(parts, t.contiguous(), group=group)
        res.append(parts)
    return res[0], res[1], res[2]
