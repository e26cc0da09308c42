"""Algorithmic work of the MSA forward (for roofline fractions).

Counts follow the method, not the implementation: intermediates (partials,
lists, block scores) are excluded.

* index FLOPs: every (query, group) with more causal blocks than k scores the
  d_idx-dim index query against the B_k keys of each non-local causal block:
  2 * G * d_idx * B_k * (nb(t) - 1).  Queries with nb(t) <= k need no scores.
* main FLOPs: 4 * H * d * att(t) per query (QK^T and PV), att(t) the number of
  tokens it attends: t+1 while nb(t) <= k, else (k-1)*B_k + (t mod B_k) + 1.
* prefill bytes: q, k, v, q_idx, k_idx read once and the output written once.
* decode bytes: the whole index-key cache once, plus the K and V rows of the
  selected blocks, plus q / q_idx / out.
"""
from __future__ import annotations

from typing import Dict, Sequence


def _prefill_seq(S: int, T: int, H: int, G: int, d: int, d_idx: int, B_k: int, k: int):
    idx = 0
    main = 0
    for i in range(T):
        p = S - T + i
        nb = p // B_k + 1
        if nb > k:
            idx += 2 * G * d_idx * B_k * (nb - 1)
            att = (k - 1) * B_k + (p % B_k) + 1
        else:
            att = p + 1
        main += 4 * H * d * att
    return idx, main


def _prefill_seq_fast(S: int, T: int, H: int, G: int, d: int, d_idx: int, B_k: int, k: int):
    """Closed-form sums of _prefill_seq over whole blocks (same result)."""
    idx = 0
    main = 0
    p0 = S - T
    # iterate by block to stay O(nb)
    p = p0
    while p < S:
        blk = p // B_k
        end = min(S, (blk + 1) * B_k)
        n = end - p
        nb = blk + 1
        first_in = p % B_k
        if nb > k:
            idx += 2 * G * d_idx * B_k * (nb - 1) * n
            # att = (k-1)B_k + (p mod B_k) + 1 for p in [p, end)
            s_att = n * ((k - 1) * B_k + 1) + (first_in + first_in + n - 1) * n // 2
        else:
            s_att = (p + 1 + end) * n // 2
        main += 4 * H * d * s_att
        p = end
    return idx, main


def prefill_work(S_lens: Sequence[int], T_lens: Sequence[int], H: int, G: int, d: int, d_idx: int,
                 B_k: int, k: int) -> Dict[str, float]:
    idx = main = 0
    for S, T in zip(S_lens, T_lens):
        a, b = _prefill_seq_fast(S, T, H, G, d, d_idx, B_k, k)
        idx += a
        main += b
    T_tot, S_tot = sum(T_lens), sum(S_lens)
    nbytes = 2 * (T_tot * H * d + 2 * S_tot * G * d + T_tot * G * d_idx + S_tot * d_idx + T_tot * H * d)
    return {"index_flops": float(idx), "main_flops": float(main), "flops": float(idx + main),
            "bytes": float(nbytes)}


def dense_work(S_lens: Sequence[int], T_lens: Sequence[int], H: int, d: int) -> float:
    """FLOPs of dense causal attention (every key <= the query position)."""
    fl = 0
    for S, T in zip(S_lens, T_lens):
        p0 = S - T
        fl += 4 * H * d * ((p0 + 1 + S) * T // 2)
    return float(fl)


def decode_work(L_lens: Sequence[int], H: int, G: int, d: int, d_idx: int, B_k: int, k: int) -> Dict[str, float]:
    idx_bytes = 2 * sum(L_lens) * d_idx
    kv_bytes = 0
    for L in L_lens:
        nb = (L - 1) // B_k + 1
        nsel = min(k, nb)
        toks = min(L, (nsel - 1) * B_k + ((L - 1) % B_k) + 1)
        kv_bytes += 2 * 2 * toks * G * d
    small = 2 * len(L_lens) * (2 * H * d + G * d_idx)
    flops = sum(2 * G * d_idx * L for L in L_lens) + 4 * H * d * sum(
        min(L, (min(k, (L - 1) // B_k + 1) - 1) * B_k + ((L - 1) % B_k) + 1) for L in L_lens)
    return {"bytes": float(idx_bytes + kv_bytes + small), "index_bytes": float(idx_bytes),
            "kv_bytes": float(kv_bytes), "flops": float(flops)}
