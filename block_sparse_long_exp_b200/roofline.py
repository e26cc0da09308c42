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
* training kernels, over the same supports (att(t) keys per query and head):
  backward 10 * d per (query, head, key) (S = q.k, dP = dO.v, dq += dS k,
  dk += dS q, dv += P dO: 2.5x the main FLOPs); the KL target 2 * d per head
  score plus 2 * d_idx for the index score per (query, group, key); its
  gradient that plus 4 * d_idx (dq_idx and dk_idx).  Exponentials and
  logarithms are not counted.
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


def training_work(S_lens: Sequence[int], T_lens: Sequence[int], H: int, G: int, d: int, d_idx: int,
                  B_k: int, k: int) -> Dict[str, float]:
    """FLOPs of the Main Branch backward and of the KL target and its gradient
    over the selected supports of a prefill layer."""
    main = prefill_work(S_lens, T_lens, H, G, d, d_idx, B_k, k)["main_flops"]
    pairs = main / (4 * H * d)            # attended (query, key) pairs of one head
    return {"pairs": pairs, "backward_flops": 10.0 * H * d * pairs,
            "kl_flops": pairs * (2.0 * H * d + 2.0 * G * d_idx),
            # on the tensor cores: the teacher scores q . k and the raw index scores q_idx . k_idx
            "kl_tensor_flops": pairs * (2.0 * H * d + 2.0 * G * d_idx),
            "kl_exps": pairs * H,                        # one exponential per head and attended pair
            "kl_grad_flops": pairs * (2.0 * H * d + 6.0 * G * d_idx),
            # the gradient's products on the CUDA cores: dq_idx and dk_idx, 2 d_idx each
            "kl_grad_alu_flops": pairs * 4.0 * G * d_idx}


def alu_fp32_tflops(sms: int = 148, lanes: int = 128, mhz: float = 1965.0) -> float:
    """Peak fp32 FMA rate of the CUDA cores (two FLOPs per lane per clock):
    B200 has 148 SMs of 128 fp32 lanes, clocks.max.sm 1965 MHz: 74.4 TFLOP/s."""
    return sms * lanes * 2.0 * mhz * 1e6 / 1e12


def mufu_gexps(sms: int = 148, per_clk: int = 16, mhz: float = 1965.0) -> float:
    """Peak exponential rate of the special-function units: 16 ex2 per clock
    per SM (the rate measured on B200 for every ex2 form), 148 SMs at
    clocks.max.sm 1965 MHz: 4653 G exponentials/s."""
    return sms * per_clk * mhz * 1e6 / 1e9


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


def tile_split(sel, cu_q_host: Sequence[int], cu_k_host: Sequence[int], H: int, G: int, d: int, B_k: int,
               theta: int, q_chunk: int = 0) -> Dict[str, float]:
    """Algorithmic work of each main-branch kernel for one prefill call.

    Re-derives, with torch ops on the selection `sel` [T, G, k] (device or
    host), which selections the query tiles cover: a tile is UQ = 2 x 128 /
    max(H/G, 8) consecutive rows of one pass that lie in one sequence, and a
    block chosen by >= theta of its queries (for one group) is covered.
    Returns the FLOPs of the covered selections (tile kernel) and of the rest
    (KV-outer kernel), counted as 4 * d * (H/G) per attended (row, key), and
    the bytes the combine must move: the merged slots' partials (f16) and
    log-sum-exps read, and the merged outputs (bf16) and log-sum-exps written;
    also the MMA work the tile kernel issues (whole 128-row tiles per dense
    block, including the rows of queries that did not choose the block).
    """
    import torch

    T, _, k = sel.shape
    Hg = H // G
    UQ = 2 * (128 // max(Hg, 8))
    dev = sel.device
    # query position and local block of every row
    pos = torch.empty(T, dtype=torch.int64)
    for b in range(len(cu_q_host) - 1):
        Tb, Sb = cu_q_host[b + 1] - cu_q_host[b], cu_k_host[b + 1] - cu_k_host[b]
        pos[cu_q_host[b]:cu_q_host[b + 1]] = torch.arange(Sb - Tb, Sb)
    seq = torch.empty(T, dtype=torch.int64)
    for b in range(len(cu_q_host) - 1):
        seq[cu_q_host[b]:cu_q_host[b + 1]] = b
    pos, seq = pos.to(dev), seq.to(dev)
    s = sel.to(torch.int64)
    valid = s >= 0
    # attended keys per (row, group, slot): whole block, or up to the position in the local block
    lb = (pos // B_k)[:, None, None]
    att = torch.where(s < lb, torch.full_like(s, B_k), (pos % B_k + 1)[:, None, None].expand_as(s))
    att = torch.where(valid, att, torch.zeros_like(att))
    covered = torch.zeros_like(valid)
    tile_blocks = 0          # (unit, dense block, 128-row MMA tile) triples the tile kernel runs
    RQ = max(Hg, 8)
    qpt = 128 // RQ
    if theta > 0:
        rows = T if q_chunk <= 0 else q_chunk
        for t0 in range(0, T, rows):
            t1 = min(T, t0 + rows)
            n = t1 - t0
            nu = (n + UQ - 1) // UQ
            pad = nu * UQ - n
            sp = torch.nn.functional.pad(s[t0:t1], (0, 0, 0, 0, 0, pad), value=-1)
            sq = torch.nn.functional.pad(seq[t0:t1], (0, pad), value=-1)
            one = sq.view(nu, UQ)
            last = torch.tensor([min(UQ, n - u * UQ) - 1 for u in range(nu)], device=dev)
            one_seq = one[:, 0] == one.gather(1, last[:, None])[:, 0]
            u = sp.view(nu, UQ, G, k).permute(0, 2, 1, 3).reshape(nu * G, UQ * k)
            big = torch.iinfo(torch.int64).max
            v = torch.where(u >= 0, u, torch.full_like(u, big))
            srt, _ = torch.sort(v, dim=1)
            cnt = torch.searchsorted(srt, v, right=True) - torch.searchsorted(srt, v)
            oneg = one_seq.repeat_interleave(G)
            cov = (u >= 0) & (cnt >= theta) & oneg[:, None]
            start = torch.ones_like(srt, dtype=torch.bool)
            start[:, 1:] = srt[:, 1:] != srt[:, :-1]
            runlen = torch.searchsorted(srt, srt, right=True) - torch.searchsorted(srt, srt)
            nd = (start & (runlen >= theta) & (srt != big)).sum(1).clamp(max=64) * oneg
            nq = torch.tensor([min(UQ, n - x * UQ) for x in range(nu)], device=dev).repeat_interleave(G)
            tile_blocks += int((nd * torch.where(nq > qpt, 2, 1)).sum().item())
            cov = cov.view(nu, G, UQ, k).permute(0, 2, 1, 3).reshape(nu * UQ, G, k)[:n]
            covered[t0:t1] = cov
    tile_att = (att * covered).sum().item()
    kv_att = (att * (valid & ~covered)).sum().item()
    ncov = covered.sum(-1)
    complete = (ncov > 0) & (ncov == valid.sum(-1))
    merged_slots = ((valid & ~covered).sum(-1) + (ncov > 0).to(torch.int64))[~complete]
    npairs = int((~complete).sum().item())
    comb_bytes = (merged_slots.sum().item() * Hg * (d * 2 + 4) + npairs * 8
                  + npairs * (Hg * d * 2 + Hg * 4))
    return {"tile_flops": float(4 * d * Hg * tile_att), "kv_flops": float(4 * d * Hg * kv_att),
            "tile_mma_flops": float(tile_blocks * 4 * 128 * 128 * d),
            "combine_bytes": float(comb_bytes), "combine_pairs": npairs,
            "complete_pairs": int(complete.sum().item()), "theta": theta, "tile_queries": UQ}
