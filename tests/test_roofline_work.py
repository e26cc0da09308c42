"""The algorithmic work the bench divides by (block_sparse_long_exp_b200/roofline.py),
pinned three ways on the CPU:

* the block-wise closed form against the per-token loop;
* main-branch FLOPs and decode K/V bytes against the token sets of the
  oracle's own selection (4 * d FLOPs per head and attended token; 2 * 2 * d
  bytes per group and selected token);
* the totals of the benchmark configurations against the figures derived by
  hand from the method (index FLOPs sum 2 G d_idx B_k (nb - 1) over queries
  with nb > k, main FLOPs sum 4 H d att(t), bytes of the inputs read once and
  the output written once).
"""
import numpy as np
import pytest

from block_sparse_long_exp_b200 import roofline as R
from oracle import msa_oracle as O


@pytest.mark.parametrize("S,T,B_k,k", [(1, 1, 4, 2), (9, 9, 4, 2), (37, 37, 4, 3), (37, 11, 4, 3),
                                       (300, 300, 16, 4), (300, 1, 16, 4), (129, 128, 128, 1),
                                       (5000, 4000, 128, 16)])
def test_closed_form_equals_the_token_loop(S, T, B_k, k):
    assert R._prefill_seq_fast(S, T, 8, 2, 64, 32, B_k, k) == R._prefill_seq(S, T, 8, 2, 64, 32, B_k, k)


def test_main_flops_and_decode_bytes_follow_the_oracle_selection():
    rng = np.random.default_rng(4)
    H, G, d, d_idx, B_k, k = 4, 2, 8, 3, 4, 3
    S_lens, T_lens = [23, 9, 40], [23, 9, 13]
    cu_k = np.concatenate([[0], np.cumsum(S_lens)]).tolist()
    cu_q = np.concatenate([[0], np.cumsum(T_lens)]).tolist()
    q_idx = rng.integers(-2, 3, size=(cu_q[-1], G, d_idx)).astype(np.float64)
    k_idx = rng.integers(-2, 3, size=(cu_k[-1], d_idx)).astype(np.float64)
    sel = O.index_topk(q_idx, k_idx, cu_q, cu_k, k, B_k)
    main = scored = 0
    for b in range(len(S_lens)):
        for i, pos in enumerate(O.query_positions(T_lens[b], S_lens[b])):
            t = cu_q[b] + i
            for g in range(G):
                J = O.selected_token_set([int(x) for x in sel[t, g]], int(pos), B_k)
                main += 4 * d * (H // G) * len(J)
                lb = int(pos) // B_k
                if lb + 1 > k:
                    scored += lb * B_k            # every non-local causal block is scored
    w = R.prefill_work(S_lens, T_lens, H, G, d, d_idx, B_k, k)
    assert w["main_flops"] == main
    assert w["index_flops"] == 2 * d_idx * scored
    # decode: one query at the end of each cache
    L = [1, 4, 5, 12, 13, 40]
    cu = np.concatenate([[0], np.cumsum(L)]).tolist()
    qd = rng.integers(-2, 3, size=(len(L), G, d_idx)).astype(np.float64)
    kd = rng.integers(-2, 3, size=(cu[-1], d_idx)).astype(np.float64)
    sel_d = O.index_topk(qd, kd, list(range(len(L) + 1)), cu, k, B_k)
    toks = sum(len(O.selected_token_set([int(x) for x in sel_d[b, g]], L[b] - 1, B_k))
               for b in range(len(L)) for g in range(G)) // G
    dw = R.decode_work(L, H, G, d, d_idx, B_k, k)
    assert dw["kv_bytes"] == 2 * 2 * G * d * toks
    assert dw["index_bytes"] == 2 * d_idx * sum(L)


def test_dense_flops_are_every_causal_key():
    S_lens, T_lens = [17, 30], [17, 6]
    want = sum(4 * 8 * 16 * (S - T + i + 1) for S, T in zip(S_lens, T_lens) for i in range(T))
    assert R.dense_work(S_lens, T_lens, 8, 16) == want


@pytest.mark.parametrize("T,H,G,d,d_idx,k,index_flops,main_flops,gbytes,dense_flops", [
    (4096, 8, 2, 64, 32, 8, 0.98e9, 7.12e9, 0.0113, 1.72e10),
    (32768, 64, 4, 128, 64, 16, 2.73e11, 2.07e12, 1.16, 1.76e13),
    (131072, 64, 4, 128, 64, 16, 4.39e12, 8.46e12, 4.65, 2.82e14),
    (1048576, 64, 4, 128, 64, 16, 2.81e14, 6.81e13, 37.2, 1.80e16),
])
def test_configuration_totals(T, H, G, d, d_idx, k, index_flops, main_flops, gbytes, dense_flops):
    w = R.prefill_work([T], [T], H, G, d, d_idx, 128, k)
    assert w["index_flops"] == pytest.approx(index_flops, rel=5e-3)
    assert w["main_flops"] == pytest.approx(main_flops, rel=5e-3)
    assert w["bytes"] / 1e9 == pytest.approx(gbytes, rel=5e-3)
    assert R.dense_work([T], [T], H, d) == pytest.approx(dense_flops, rel=5e-3)


def test_pages_compute_ratio_at_1m():
    """The pages report per-token attention compute at 1M tokens 28.4x below
    dense GQA (pnsm.cn sec. 9; yhxrc.cn sec. 二) for 64 query heads, 4 KV heads,
    B_k = 128, k = 16.  The work accounting reproduces it, index branch
    included, when the index head has d_idx = 128 (the pages do not state
    d_idx); with the d_idx = 64 used here the ratio is about 51.5."""
    N = 1 << 20
    dense = R.dense_work([N], [N], 64, 128)
    w128 = R.prefill_work([N], [N], 64, 4, 128, 128, 128, 16)
    assert dense / (w128["index_flops"] + w128["main_flops"]) == pytest.approx(28.4, rel=1e-2)
    w64 = R.prefill_work([N], [N], 64, 4, 128, 64, 128, 16)
    assert dense / (w64["index_flops"] + w64["main_flops"]) == pytest.approx(51.5, rel=1e-2)


def test_training_flops_follow_the_oracle_selection():
    # per attended (query, head, key): 10 d for the backward; per (query, group,
    # key): 2 d per head of the group and 2 d_idx for the KL, 4 d_idx more for
    # its gradient; the key sets are the oracle's selected token sets
    rng = np.random.default_rng(6)
    H, G, d, d_idx, B_k, k = 6, 2, 8, 5, 4, 2
    S_lens, T_lens = [30, 7, 19], [30, 7, 4]
    cu_k = np.concatenate([[0], np.cumsum(S_lens)]).tolist()
    cu_q = np.concatenate([[0], np.cumsum(T_lens)]).tolist()
    q_idx = rng.integers(-2, 3, size=(cu_q[-1], G, d_idx)).astype(np.float64)
    k_idx = rng.integers(-2, 3, size=(cu_k[-1], d_idx)).astype(np.float64)
    sel = O.index_topk(q_idx, k_idx, cu_q, cu_k, k, B_k)
    bwd = kl = klg = 0
    for b in range(len(S_lens)):
        for i, pos in enumerate(O.query_positions(T_lens[b], S_lens[b])):
            t = cu_q[b] + i
            for g in range(G):
                n = len(O.selected_token_set([int(x) for x in sel[t, g]], int(pos), B_k))
                bwd += 10 * d * (H // G) * n
                kl += n * (2 * d * (H // G) + 2 * d_idx)
                klg += n * (2 * d * (H // G) + 6 * d_idx)
    tw = R.training_work(S_lens, T_lens, H, G, d, d_idx, B_k, k)
    assert tw["backward_flops"] == bwd
    assert tw["kl_flops"] == kl and tw["kl_grad_flops"] == klg
    assert tw["backward_flops"] == 2.5 * R.prefill_work(S_lens, T_lens, H, G, d, d_idx, B_k, k)["main_flops"]


def test_cuda_core_peak():
    # 148 SMs x 128 fp32 lanes x 2 FLOPs (one FMA) x 1965 MHz
    assert R.alu_fp32_tflops() == pytest.approx(74.44992, rel=1e-9)
