"""Seeded synthetic workloads for the MSA layer.

This module only draws random inputs and states their shapes; it holds none of
the method's arithmetic.  It is the one module that both the CUDA path's tests /
bench and the CPU oracle's tests use.

Recipe (shapes from the MSA pages' 109B model: 64 query heads, 4 KV heads,
128-token blocks, k = 16, i.e. a 2048-token budget per query):

* Q, K, V: bf16 drawn from N(0, 1).
* index q / index k: integers drawn uniformly from {-4, ..., 4}, stored as bf16
  (exact), so every index score is an integer and fp32 accumulation is exact.
* "hot" blocks: round(hot_frac * nb) block ids per sequence, drawn without
  replacement; every index-key entry inside them is multiplied by 3 (exact in
  bf16), so many queries select them (skewed block popularity).
* decode: per-sequence cache lengths drawn uniformly from [L_min, L_max].

All draws come from one ``torch.Generator`` seeded per workload, on the device
the tensors are created on (CPU draws and CUDA draws differ for the same seed;
each test states which it uses).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill" or "decode"
    H: int
    G: int
    d: int
    d_idx: int
    B_k: int
    k: int
    seed: int
    T: int = 0           # prefill: tokens of the single sequence (T == S)
    batch: int = 1
    L_min: int = 0       # decode: cache length range (inclusive)
    L_max: int = 0
    hot_frac: float = 0.0

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


WORKLOADS: Dict[str, Workload] = {
    w.name: w for w in [
        Workload("tiny_n4096", "prefill", H=8, G=2, d=64, d_idx=32, B_k=128, k=8,
                 seed=0, T=4096),
        Workload("prefill_n32768", "prefill", H=64, G=4, d=128, d_idx=64, B_k=128,
                 k=16, seed=1, T=32768),
        Workload("prefill_n131072_hot2", "prefill", H=64, G=4, d=128, d_idx=64,
                 B_k=128, k=16, seed=2, T=131072, hot_frac=0.02),
        Workload("decode_b32_l128k_1m_hot2", "decode", H=64, G=4, d=128, d_idx=64,
                 B_k=128, k=16, seed=3, batch=32, L_min=131072, L_max=1048576,
                 hot_frac=0.02),
        Workload("prefill_n1048576_hot2", "prefill", H=64, G=4, d=128, d_idx=64,
                 B_k=128, k=16, seed=4, T=1048576, hot_frac=0.02),
        # a smaller decode batch of the same shape for profiler captures: its
        # index keys (~0.4 GB) still exceed L2, its K/V caches are ~6 GB
        Workload("decode_b4_l512k_1m_hot2", "decode", H=64, G=4, d=128, d_idx=64,
                 B_k=128, k=16, seed=5, batch=4, L_min=524288, L_max=1048576,
                 hot_frac=0.02),
    ]
}


def _randn_bf16(shape, gen: torch.Generator, device, chunk: int = 1 << 26) -> torch.Tensor:
    """N(0,1) bf16, drawn in chunks so that huge tensors do not need an fp32 copy."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        flat[s:e] = torch.randn(e - s, generator=gen, device=device,
                                dtype=torch.float32).to(torch.bfloat16)
    return out


def _randint_bf16(shape, lo: int, hi: int, gen: torch.Generator, device,
                  chunk: int = 1 << 26) -> torch.Tensor:
    """Integers uniform in [lo, hi] (inclusive), stored as bf16."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        flat[s:e] = torch.randint(lo, hi + 1, (e - s,), generator=gen, device=device,
                                  dtype=torch.int32).to(torch.bfloat16)
    return out


def _make_hot(k_idx: torch.Tensor, cu: List[int], B_k: int, frac: float,
              gen: torch.Generator) -> List[List[int]]:
    """Scale the index keys of round(frac * nb) random blocks per sequence by 3."""
    hot_all = []
    for b in range(len(cu) - 1):
        n = cu[b + 1] - cu[b]
        nb = -(-n // B_k)
        n_hot = int(round(frac * nb))
        hot = []
        if n_hot > 0:
            perm = torch.randperm(nb, generator=gen, device=gen.device)[:n_hot]
            hot = sorted(int(x) for x in perm.cpu())
            for blk in hot:
                r0 = cu[b] + blk * B_k
                r1 = min(cu[b] + (blk + 1) * B_k, cu[b + 1])
                k_idx[r0:r1] *= 3
        hot_all.append(hot)
    return hot_all


def seq_lengths(w: Workload, gen: Optional[torch.Generator] = None) -> List[int]:
    if w.kind == "prefill":
        return [w.T] * w.batch
    assert gen is not None
    L = torch.randint(w.L_min, w.L_max + 1, (w.batch,), generator=gen,
                      device=gen.device, dtype=torch.int64)
    return [int(x) for x in L.cpu()]


def make_inputs(w: Workload, device="cpu", T_override: Optional[int] = None,
                lengths: Optional[List[int]] = None) -> Dict[str, object]:
    """Draw one workload's inputs on ``device``.

    ``T_override`` shrinks a prefill workload to a shorter sequence with the same
    heads and dims (for parity tests); ``lengths`` gives explicit per-sequence
    key lengths (prefill: T_b = S_b; decode: one query per sequence).

    Returns a dict of tensors: q [T,H,d], k/v [S,G,d], q_idx [T,G,d_idx],
    k_idx [S,d_idx] (all bf16), cu_q / cu_k int32 [B+1] (on ``device``) and the
    host lists ``cu_q_host`` / ``cu_k_host`` and ``hot_blocks``.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    if lengths is None:
        if w.kind == "prefill":
            lengths = [T_override or w.T] * w.batch
        else:
            lengths = seq_lengths(w, gen)
    S_lens = list(lengths)
    T_lens = S_lens if w.kind == "prefill" else [1] * len(S_lens)
    cu_k = [0]
    for n in S_lens:
        cu_k.append(cu_k[-1] + n)
    cu_q = [0]
    for n in T_lens:
        cu_q.append(cu_q[-1] + n)
    T, S = cu_q[-1], cu_k[-1]
    q = _randn_bf16((T, w.H, w.d), gen, device)
    k = _randn_bf16((S, w.G, w.d), gen, device)
    v = _randn_bf16((S, w.G, w.d), gen, device)
    q_idx = _randint_bf16((T, w.G, w.d_idx), -4, 4, gen, device)
    k_idx = _randint_bf16((S, w.d_idx), -4, 4, gen, device)
    hot = _make_hot(k_idx, cu_k, w.B_k, w.hot_frac, gen)
    return {
        "q": q, "k": k, "v": v, "q_idx": q_idx, "k_idx": k_idx,
        "cu_q": torch.tensor(cu_q, dtype=torch.int32, device=device),
        "cu_k": torch.tensor(cu_k, dtype=torch.int32, device=device),
        "cu_q_host": cu_q, "cu_k_host": cu_k, "hot_blocks": hot,
    }


def sample_rows(T_lens: List[int], B_k: int, k: int, n: int, seed: int,
                hot_blocks: Optional[List[List[int]]] = None) -> List[int]:
    """Seeded sample of query rows for parity at sizes the oracle cannot finish
    in full: n random rows plus the boundary rows t in {0, B_k-1, B_k, k*B_k-1,
    k*B_k, k*B_k+1, T-1} of every sequence and the first row after each hot
    block."""
    g = torch.Generator().manual_seed(seed)
    rows = set()
    off = 0
    for b, Tb in enumerate(T_lens):
        for t in (0, B_k - 1, B_k, k * B_k - 1, k * B_k, k * B_k + 1, Tb - 1):
            if 0 <= t < Tb:
                rows.add(off + t)
        if hot_blocks is not None:
            for blk in hot_blocks[b]:
                t = (blk + 1) * B_k
                if t < Tb:
                    rows.add(off + t)
        off += Tb
    total = off
    m = min(n, total)
    rnd = torch.randperm(total, generator=g)[:m]
    rows.update(int(x) for x in rnd)
    return sorted(rows)
