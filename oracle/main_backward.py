"""Plain fp64 CPU oracle of the Main Branch's backward: the gradients of the
sparse attention output with respect to q, k and v, for a given selection.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this module: only the tests may use it.  It shares no code with the CUDA path.

What it computes (the pages train MSA end to end, so the attention over the
selected blocks is differentiated like any softmax attention; [yifor] "設計核心"
item 2 and [pnsm] sec. 2 fix the forward this differentiates): for query t,
head h of group g and its support J (the selected blocks' tokens cut at the
query, or every causal token in the dense form),
    s_j = sm_scale q_h . k_j,  P_j = exp(s_j - lse_h),  o_h = sum_j P_j v_j,
and for an upstream gradient dO = d loss / d o_h,
    dP_j = dO . v_j,   D = sum_j P_j dP_j = dO . o_h,   dS_j = P_j (dP_j - D),
    dq_h      = sm_scale sum_j dS_j k_j,
    dk_j     += sm_scale dS_j q_h,     dv_j += P_j dO     (summed over every
                                                           (t, h) that reaches j).
The selection itself is not differentiated (it is a top-k).
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

from oracle import msa_oracle as O

__all__ = ["main_branch_backward"]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def main_branch_backward(q, k, v, sel, dout, cu_q, cu_k, B_k: int, sm_scale: float,
                         dense: bool = False) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """dq [T, H, d], dk [S, G, d], dv [S, G, d] for the upstream gradient dout
    [T, H, d] (q [T, H, d], k / v [S, G, d], sel [T, G, k]; packed sequences
    whose queries are their last T_b tokens)."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    T, H, d = q.shape
    G = k.shape[1]
    Hg = H // G
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(len(cu_q) - 1):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
        for i, pos in enumerate(O.query_positions(q1 - q0, k1 - k0)):
            t = q0 + i
            for g in range(G):
                if dense:
                    J = np.arange(int(pos) + 1)
                else:
                    J = O.selected_token_set([int(x) for x in sel[t, g]], int(pos), B_k)
                Kj, Vj = k[k0 + J, g], v[k0 + J, g]
                for h in range(g * Hg, (g + 1) * Hg):
                    s = sm_scale * (Kj @ q[t, h])
                    P = np.exp(s - s.max())
                    P /= P.sum()
                    o = P @ Vj
                    dP = Vj @ dout[t, h]
                    dS = P * (dP - dout[t, h] @ o)
                    dq[t, h] = sm_scale * (dS @ Kj)
                    # J holds each token once, so indexed += adds every row exactly once
                    dk[k0 + J, g] += sm_scale * np.outer(dS, q[t, h])
                    dv[k0 + J, g] += np.outer(P, dout[t, h])
    return dq, dk, dv
