"""Plain fp64 CPU oracle of MSA's index-alignment target: the KL term that
trains the Index Branch against the Main Branch's attention, its gradient
with respect to the index query and key, and the share of the attention
weight that the selected blocks hold.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this module: only the tests may use it.  It shares no code with the CUDA path.
No kernel computes this target yet; this oracle comes first, pinned, so that
the kernel that follows can be held to it.

Sources (web pages about MSA; cited by title / address and section):

* [pnsm]  "MiniMax Sparse Attention：一篇读懂百万上下文时代的稀疏注意力工程化路线"
  (pnsm.cn), sec. 4 "训练难点：Top-k 不可导，Indexer 怎么学会选对 block": the
  Index Branch's distribution is pulled by a KL divergence towards the Main
  Branch's attention distribution on the selected support, and the gradient
  of that term is detached from the backbone, reaching only the index
  query / key projections; sec. 5 "Indexer warmup": before sparse routing,
  the Main Branch attends densely and the Index Branch aligns to the whole
  attention distribution; the glossary "术语与概念速查" (rows "KL alignment
  loss", "gradient detach", "indexer warmup").
* [yhxrc] M3 / MSA comparison article (yhxrc.cn), sec. 二 "MSA是怎么做的": the
  Main Branch's attention is the teacher, the alignment keeps running on the
  chosen blocks after warmup, and the chosen blocks are reported to hold most
  of the Main Branch's attention weight (a monitored quantity).

Readings where the pages are silent (each is listed in the design notes):

* granularity: tokens.  The support J(t, g) is the main branch's token set
  (the selected blocks cut causally at the query) or, in the warmup form,
  every causal token [0, pos];
* teacher P: the mean, over the group's H/G query heads, of their attention
  distributions over J (the index branch has one query head per group; a
  mixture of distributions is a distribution);
* student Q: softmax over J of the index scores s_j = <q_idx[t,g], k_idx[j]>
  times a scale tau (an argument: the selection does not depend on a positive
  scale, the distribution does);
* divergence: KL(P || Q) = sum_j P_j (log P_j - log Q_j), with 0 log 0 = 0,
  one value per (query, group); the loss is their sum (a mean is that sum
  over T * G);
* detach: P is a constant.  With student logits z_j = tau * s_j,
  d KL / d z_j = Q_j - P_j, so
      dq_idx[t, g] = tau * sum_j (Q_j - P_j) k_idx[j],
      dk_idx[j]   += tau * (Q_j - P_j) q_idx[t, g]   (summed over t, g).
"""
from __future__ import annotations

from typing import Sequence, Tuple

import numpy as np

from oracle import msa_oracle as O

__all__ = [
    "support",
    "teacher_distribution",
    "student_log_distribution",
    "kl_divergence",
    "index_kl_rows",
    "index_kl_loss_and_grad",
    "selected_attention_mass",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def support(blocks: Sequence[int], pos: int, B_k: int, dense: bool = False) -> np.ndarray:
    """J(t, g): the main branch's token set, or every causal token when dense
    (the warmup form, [pnsm] sec. 5)."""
    if dense:
        return np.arange(pos + 1, dtype=np.int64)
    return O.selected_token_set(blocks, pos, B_k)


def teacher_distribution(q_tg, K_J, sm_scale: float) -> np.ndarray:
    """P over J: the mean of the group's heads' softmax distributions of
    sm_scale * q_h . k_j ([pnsm] sec. 4: the Main Branch's attention on the
    support is the target)."""
    s = sm_scale * (_f64(q_tg) @ _f64(K_J).T)          # [Hg, |J|]
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return (e / e.sum(axis=1, keepdims=True)).mean(axis=0)


def student_log_distribution(q_idx_tg, k_idx_J, tau: float) -> np.ndarray:
    """log Q over J: log-softmax of tau times the raw index scores."""
    z = tau * (_f64(k_idx_J) @ _f64(q_idx_tg))          # [|J|]
    m = z.max()
    return z - (m + np.log(np.exp(z - m).sum()))


def kl_divergence(P, logQ) -> float:
    """KL(P || Q) = sum_j P_j (log P_j - log Q_j); terms with P_j = 0 are 0."""
    P = _f64(P)
    nz = P > 0
    return float(np.sum(P[nz] * (np.log(P[nz]) - _f64(logQ)[nz])))


def _rows_of(cu_q, cu_k, t: int) -> Tuple[int, int, int]:
    """(sequence, absolute position, first key row) of packed query row t."""
    cu_q = np.asarray(cu_q, dtype=np.int64)
    cu_k = np.asarray(cu_k, dtype=np.int64)
    b = int(np.searchsorted(cu_q, t, side="right") - 1)
    T_b = int(cu_q[b + 1] - cu_q[b])
    S_b = int(cu_k[b + 1] - cu_k[b])
    return b, S_b - T_b + (t - int(cu_q[b])), int(cu_k[b])


def index_kl_rows(q, k, q_idx, k_idx, sel, cu_q, cu_k, rows: Sequence[int], B_k: int,
                  sm_scale: float, tau: float, dense: bool = False) -> np.ndarray:
    """KL(P || Q) for every listed query row and group: kl [len(rows), G].

    q [T, H, d], k [S, G, d], q_idx [T, G, d_idx], k_idx [S, d_idx], sel [T, G, k]
    (packed sequences; the queries of a sequence are its last T_b tokens)."""
    q, k, q_idx, k_idx = _f64(q), _f64(k), _f64(q_idx), _f64(k_idx)
    H, G = q.shape[1], k.shape[1]
    Hg = H // G
    out = np.zeros((len(rows), G))
    for r, t in enumerate(rows):
        _, pos, k0 = _rows_of(cu_q, cu_k, t)
        for g in range(G):
            J = support([int(x) for x in sel[t, g]], pos, B_k, dense) + k0
            P = teacher_distribution(q[t, g * Hg:(g + 1) * Hg], k[J, g], sm_scale)
            logQ = student_log_distribution(q_idx[t, g], k_idx[J], tau)
            out[r, g] = kl_divergence(P, logQ)
    return out


def index_kl_loss_and_grad(q, k, q_idx, k_idx, sel, cu_q, cu_k, B_k: int, sm_scale: float,
                           tau: float, dense: bool = False) -> Tuple[float, np.ndarray, np.ndarray]:
    """The loss sum_{t,g} KL(P || Q) over every query row, and its gradient with
    respect to q_idx [T, G, d_idx] and k_idx [S, d_idx] with the teacher held
    constant ([pnsm] sec. 4 "gradient detach")."""
    q, k, q_idx, k_idx = _f64(q), _f64(k), _f64(q_idx), _f64(k_idx)
    T, H, _ = q.shape
    G = k.shape[1]
    Hg = H // G
    loss = 0.0
    dq = np.zeros_like(q_idx)
    dk = np.zeros_like(k_idx)
    for t in range(T):
        _, pos, k0 = _rows_of(cu_q, cu_k, t)
        for g in range(G):
            J = support([int(x) for x in sel[t, g]], pos, B_k, dense) + k0
            P = teacher_distribution(q[t, g * Hg:(g + 1) * Hg], k[J, g], sm_scale)
            logQ = student_log_distribution(q_idx[t, g], k_idx[J], tau)
            loss += kl_divergence(P, logQ)
            w = tau * (np.exp(logQ) - P)                 # d KL / d s_j
            dq[t, g] += w @ k_idx[J]
            np.add.at(dk, J, np.outer(w, q_idx[t, g]))
    return loss, dq, dk


def selected_attention_mass(q, k, sel, cu_q, cu_k, rows: Sequence[int], B_k: int,
                            sm_scale: float) -> np.ndarray:
    """Share of each head's dense causal attention weight that falls on the
    selected tokens ([yhxrc] sec. 二 reports this share as a monitor):
    mass[r, h] = sum_{j in J} softmax_{j' <= pos}(sm_scale q_h . k_j')_j."""
    q, k = _f64(q), _f64(k)
    H, G = q.shape[1], k.shape[1]
    Hg = H // G
    out = np.zeros((len(rows), H))
    for r, t in enumerate(rows):
        _, pos, k0 = _rows_of(cu_q, cu_k, t)
        for h in range(H):
            g = h // Hg
            s = sm_scale * (k[k0:k0 + pos + 1, g] @ q[t, h])
            p = np.exp(s - s.max())
            p /= p.sum()
            J = O.selected_token_set([int(x) for x in sel[t, g]], pos, B_k)
            out[r, h] = p[J].sum()
    return out
