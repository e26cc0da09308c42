"""Pins of the index-alignment oracle (oracle/index_kl.py) against things other
than itself (CPU only):

* brute force: the KL of every (query, group) by plain Python loops over the
  tokens (math.exp / math.log), varlen, queries that are the last T_b tokens;
* a closed form: on a two-token support both distributions are Bernoulli, and
  KL(Bern(p) || Bern(q)) = p log(p/q) + (1-p) log((1-p)/(1-q));
* zero exactly when the student equals the teacher (one head per group, index
  vectors a scaled copy of q / k), positive otherwise;
* the gradient with the teacher held constant against torch autograd in fp64
  (a separate formulation through a library routine) and against central
  finite differences of the loss;
* the warmup (dense) support equals the sparse one when every causal block is
  selected;
* the selected share of the dense attention weight equals
  exp(lse over the selected tokens - lse over all causal tokens), both from the
  main-branch oracle;
* the block-by-block split of the KL (two plain sums and an online
  log-sum-exp, the form a kernel computes) reproduces it on every row.
"""
import math

import numpy as np
import pytest
import torch

from oracle import index_kl as K
from oracle import msa_oracle as O


def _layer(seed, S_lens, T_lens, G=2, Hg=2, d=4, d_idx=3, B_k=4, k=2, int_idx=False):
    rng = np.random.default_rng(seed)
    S, T = sum(S_lens), sum(T_lens)
    cu_k = np.concatenate([[0], np.cumsum(S_lens)]).tolist()
    cu_q = np.concatenate([[0], np.cumsum(T_lens)]).tolist()
    q = rng.standard_normal((T, G * Hg, d))
    kk = rng.standard_normal((S, G, d))
    if int_idx:
        q_idx = rng.integers(-2, 3, size=(T, G, d_idx)).astype(np.float64)
        k_idx = rng.integers(-2, 3, size=(S, d_idx)).astype(np.float64)
    else:
        q_idx = rng.standard_normal((T, G, d_idx))
        k_idx = rng.standard_normal((S, d_idx))
    sel = O.index_topk(q_idx, k_idx, cu_q, cu_k, k, B_k)
    return dict(q=q, k=kk, q_idx=q_idx, k_idx=k_idx, sel=sel, cu_q=cu_q, cu_k=cu_k, B_k=B_k)


def _brute_kl(L, sm_scale, tau, dense):
    """Every (t, g) by explicit loops over tokens and coordinates."""
    q, kk, q_idx, k_idx, sel = L["q"], L["k"], L["q_idx"], L["k_idx"], L["sel"]
    cu_q, cu_k, B_k = L["cu_q"], L["cu_k"], L["B_k"]
    T, H, d = q.shape
    G = kk.shape[1]
    Hg = H // G
    out = np.zeros((T, G))
    for b in range(len(cu_q) - 1):
        T_b, S_b = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        for i in range(T_b):
            t, pos = cu_q[b] + i, S_b - T_b + i
            for g in range(G):
                chosen = {int(x) for x in sel[t, g] if x >= 0}
                J = [j for j in range(pos + 1) if dense or j // B_k in chosen]
                P = [0.0] * len(J)
                for h in range(g * Hg, (g + 1) * Hg):
                    e = [math.exp(sm_scale * sum(q[t, h, c] * kk[cu_k[b] + j, g, c] for c in range(d))) for j in J]
                    tot = sum(e)
                    for n in range(len(J)):
                        P[n] += e[n] / tot / Hg
                z = [math.exp(tau * sum(q_idx[t, g, c] * k_idx[cu_k[b] + j, c] for c in range(q_idx.shape[2])))
                     for j in J]
                zt = sum(z)
                out[t, g] = sum(P[n] * math.log(P[n] / (z[n] / zt)) for n in range(len(J)) if P[n] > 0)
    return out


@pytest.mark.parametrize("dense", [False, True])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_kl_matches_brute_force(seed, dense):
    L = _layer(seed, S_lens=[13, 1, 22], T_lens=[13, 1, 9], int_idx=(seed == 2))
    T = L["cu_q"][-1]
    got = K.index_kl_rows(L["q"], L["k"], L["q_idx"], L["k_idx"], L["sel"], L["cu_q"], L["cu_k"],
                          list(range(T)), L["B_k"], 0.5, 0.7, dense=dense)
    np.testing.assert_allclose(got, _brute_kl(L, 0.5, 0.7, dense), rtol=1e-10, atol=1e-13)
    assert np.all(got >= -1e-15)


def test_two_token_support_is_bernoulli():
    """Query at position 1, B_k = 2: the support is tokens {0, 1}."""
    rng = np.random.default_rng(5)
    Hg, d, d_idx = 3, 4, 2
    q = rng.standard_normal((2, Hg, d))
    kk = rng.standard_normal((2, 1, d))
    q_idx = rng.standard_normal((2, 1, d_idx))
    k_idx = rng.standard_normal((2, d_idx))
    sel = np.array([[[0]], [[0]]], dtype=np.int32)
    sm, tau = 0.8, 1.3
    kl = K.index_kl_rows(q, kk, q_idx, k_idx, sel, [0, 2], [0, 2], [1], 2, sm, tau)[0, 0]
    sig = lambda x: 1.0 / (1.0 + math.exp(-x))  # noqa: E731
    p = np.mean([sig(sm * float(q[1, h] @ (kk[1, 0] - kk[0, 0]))) for h in range(Hg)])
    qq = sig(tau * float(q_idx[1, 0] @ (k_idx[1] - k_idx[0])))
    want = p * math.log(p / qq) + (1 - p) * math.log((1 - p) / (1 - qq))
    assert kl == pytest.approx(want, rel=1e-12, abs=1e-15)


def test_zero_exactly_when_student_equals_teacher():
    rng = np.random.default_rng(7)
    S, d, B_k = 30, 5, 4
    q = rng.standard_normal((S, 1, d))
    kk = rng.standard_normal((S, 1, d))
    sm, tau = 0.45, 2.0
    c = math.sqrt(sm / tau)                      # tau * c^2 = sm: identical logits
    q_idx, k_idx = c * q, c * kk[:, 0]
    sel = O.index_topk(q_idx, k_idx, [0, S], [0, S], 3, B_k)
    kl = K.index_kl_rows(q, kk, q_idx, k_idx, sel, [0, S], [0, S], list(range(S)), B_k, sm, tau)
    assert np.max(np.abs(kl)) < 1e-14
    kl2 = K.index_kl_rows(q, kk, q_idx * 1.5, k_idx, sel, [0, S], [0, S], list(range(S)), B_k, sm, tau)
    assert np.all(kl2[1:] > 1e-6)                # query 0 has one token: KL = 0 there


def _torch_loss(L, sm, tau, dense, q_idx, k_idx):
    """The same loss written with torch ops; the teacher under no_grad."""
    q = torch.from_numpy(L["q"])
    kk = torch.from_numpy(L["k"])
    sel, cu_q, cu_k, B_k = L["sel"], L["cu_q"], L["cu_k"], L["B_k"]
    T, H, _ = q.shape
    G = kk.shape[1]
    Hg = H // G
    loss = torch.zeros((), dtype=torch.float64)
    for b in range(len(cu_q) - 1):
        T_b, S_b = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        for i in range(T_b):
            t, pos = cu_q[b] + i, S_b - T_b + i
            for g in range(G):
                chosen = {int(x) for x in sel[t, g] if x >= 0}
                J = torch.tensor([cu_k[b] + j for j in range(pos + 1) if dense or j // B_k in chosen])
                with torch.no_grad():
                    P = torch.softmax(sm * q[t, g * Hg:(g + 1) * Hg] @ kk[J, g].T, dim=-1).mean(0)
                logQ = torch.log_softmax(tau * k_idx[J] @ q_idx[t, g], dim=-1)
                loss = loss + torch.sum(torch.special.xlogy(P, P) - P * logQ)
    return loss


@pytest.mark.parametrize("dense", [False, True])
def test_gradient_matches_autograd_and_finite_differences(dense):
    L = _layer(11, S_lens=[17, 9], T_lens=[17, 4])
    sm, tau = 0.6, 0.9
    loss, dq, dk = K.index_kl_loss_and_grad(L["q"], L["k"], L["q_idx"], L["k_idx"], L["sel"], L["cu_q"],
                                            L["cu_k"], L["B_k"], sm, tau, dense=dense)
    qi = torch.from_numpy(L["q_idx"]).requires_grad_(True)
    ki = torch.from_numpy(L["k_idx"]).requires_grad_(True)
    tl = _torch_loss(L, sm, tau, dense, qi, ki)
    tl.backward()
    assert loss == pytest.approx(tl.item(), rel=1e-12)
    np.testing.assert_allclose(dq, qi.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, ki.grad.numpy(), rtol=1e-10, atol=1e-12)
    # central differences of the loss itself (the selection is held fixed)
    T = L["cu_q"][-1]

    def total(q_idx, k_idx):
        return K.index_kl_rows(L["q"], L["k"], q_idx, k_idx, L["sel"], L["cu_q"], L["cu_k"], list(range(T)),
                               L["B_k"], sm, tau, dense=dense).sum()
    eps = 1e-6
    for (t, g, c) in [(3, 0, 1), (20, 1, 2)]:
        a, b = L["q_idx"].copy(), L["q_idx"].copy()
        a[t, g, c] += eps
        b[t, g, c] -= eps
        fd = (total(a, L["k_idx"]) - total(b, L["k_idx"])) / (2 * eps)
        assert fd == pytest.approx(dq[t, g, c], rel=1e-6, abs=1e-8)
    for (j, c) in [(2, 0), (19, 1)]:
        a, b = L["k_idx"].copy(), L["k_idx"].copy()
        a[j, c] += eps
        b[j, c] -= eps
        fd = (total(L["q_idx"], a) - total(L["q_idx"], b)) / (2 * eps)
        assert fd == pytest.approx(dk[j, c], rel=1e-6, abs=1e-8)


def test_dense_support_equals_sparse_when_everything_is_selected():
    L = _layer(3, S_lens=[20, 7], T_lens=[20, 7], k=8, B_k=4)      # nb <= 5 <= k
    T = L["cu_q"][-1]
    args = (L["q"], L["k"], L["q_idx"], L["k_idx"], L["sel"], L["cu_q"], L["cu_k"], list(range(T)), L["B_k"], 0.5, 1.0)
    np.testing.assert_allclose(K.index_kl_rows(*args, dense=False), K.index_kl_rows(*args, dense=True),
                               rtol=0, atol=1e-15)
    L2 = _layer(3, S_lens=[20, 7], T_lens=[20, 7], k=2, B_k=4)     # now the supports differ
    args2 = (L2["q"], L2["k"], L2["q_idx"], L2["k_idx"], L2["sel"], L2["cu_q"], L2["cu_k"], list(range(T)),
             L2["B_k"], 0.5, 1.0)
    assert not np.allclose(K.index_kl_rows(*args2, dense=False), K.index_kl_rows(*args2, dense=True))


def test_selected_mass_is_the_lse_ratio():
    L = _layer(9, S_lens=[26, 11], T_lens=[26, 5], k=3, B_k=4)
    T = L["cu_q"][-1]
    rows = list(range(T))
    mass = K.selected_attention_mass(L["q"], L["k"], L["sel"], L["cu_q"], L["cu_k"], rows, L["B_k"], 0.7)
    v = np.zeros_like(L["k"])
    _, lse_sel = O.msa_forward_rows(L["q"], L["k"], v, L["sel"], L["cu_q"], L["cu_k"], rows, L["B_k"], 0.7)
    every = np.tile(np.arange(L["sel"].shape[2] * 10, dtype=np.int32)[None, None, :], (T, L["k"].shape[1], 1))
    _, lse_all = O.msa_forward_rows(L["q"], L["k"], v, every, L["cu_q"], L["cu_k"], rows, L["B_k"], 0.7)
    np.testing.assert_allclose(mass, np.exp(lse_sel - lse_all), rtol=1e-12, atol=0)
    assert np.all(mass <= 1 + 1e-12) and np.all(mass > 0)
    # queries whose causal blocks all fit in k hold all of the weight
    pos_small = [t for t in rows if t < 3 * L["B_k"]]
    np.testing.assert_allclose(mass[pos_small], 1.0, rtol=0, atol=1e-12)


def test_block_split_reproduces_the_kl():
    """KL = sum P log P - sum P z + log sum exp z over the support, each sum taken
    block by block (two plain sums and one (max, sum) pair per block) and merged:
    the split a kernel uses, checked against the oracle on every row."""
    L = _layer(21, S_lens=[33, 18], T_lens=[33, 7], G=2, Hg=3, k=3, B_k=4)
    sm, tau = 0.55, 0.8
    T = L["cu_q"][-1]
    want = K.index_kl_rows(L["q"], L["k"], L["q_idx"], L["k_idx"], L["sel"], L["cu_q"], L["cu_k"], list(range(T)),
                           L["B_k"], sm, tau)
    H, G = L["q"].shape[1], L["k"].shape[1]
    Hg = H // G
    for t in range(T):
        b = int(np.searchsorted(L["cu_q"], t, side="right") - 1)
        T_b, S_b = L["cu_q"][b + 1] - L["cu_q"][b], L["cu_k"][b + 1] - L["cu_k"][b]
        pos, k0 = S_b - T_b + (t - L["cu_q"][b]), L["cu_k"][b]
        for g in range(G):
            J = O.selected_token_set([int(x) for x in L["sel"][t, g]], pos, L["B_k"]) + k0
            s = sm * L["q"][t, g * Hg:(g + 1) * Hg] @ L["k"][J, g].T          # [Hg, |J|]
            lse_h = np.log(np.exp(s).sum(axis=1))                            # the forward's lse over J
            A = Bsum = 0.0
            m_z, l_z = -np.inf, 0.0
            for blk in sorted({int(j - k0) // L["B_k"] for j in J}):
                cols = [i for i, j in enumerate(J) if (j - k0) // L["B_k"] == blk]
                Pbar = np.exp(s[:, cols] - lse_h[:, None]).mean(axis=0)
                z = tau * L["k_idx"][J[cols]] @ L["q_idx"][t, g]
                A += float(np.sum(Pbar * np.log(Pbar)))
                Bsum += float(np.sum(Pbar * z))
                m_new = max(m_z, float(z.max()))
                l_z = l_z * math.exp(m_z - m_new) + float(np.exp(z - m_new).sum())
                m_z = m_new
            assert A - Bsum + (m_z + math.log(l_z)) == pytest.approx(want[t, g], rel=1e-10, abs=1e-12)
