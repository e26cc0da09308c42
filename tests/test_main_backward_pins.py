"""Pins of the Main Branch backward oracle (oracle/main_backward.py) against
things other than itself (CPU only):

* torch autograd in fp64 through softmax attention written with an explicit
  token mask built from the selection by loops (a separate formulation through
  a library routine), sparse and dense supports, varlen, last-T_b queries;
* central finite differences of a scalar loss sum(out * W) on a few
  coordinates of q, k and v;
* a closed form: a query whose support is one token has P = 1, so its dq is
  0, the key gets nothing from it and the value gets dO.
"""
import numpy as np
import pytest
import torch

from oracle import main_backward as B
from oracle import msa_oracle as O


def _layer(seed, S_lens, T_lens, G=2, Hg=2, d=4, d_idx=3, B_k=4, k=2):
    rng = np.random.default_rng(seed)
    S, T = sum(S_lens), sum(T_lens)
    cu_k = np.concatenate([[0], np.cumsum(S_lens)]).tolist()
    cu_q = np.concatenate([[0], np.cumsum(T_lens)]).tolist()
    q = rng.standard_normal((T, G * Hg, d))
    kk = rng.standard_normal((S, G, d))
    v = rng.standard_normal((S, G, d))
    q_idx = rng.standard_normal((T, G, d_idx))
    k_idx = rng.standard_normal((S, d_idx))
    sel = O.index_topk(q_idx, k_idx, cu_q, cu_k, k, B_k)
    dout = rng.standard_normal((T, G * Hg, d))
    return dict(q=q, k=kk, v=v, sel=sel, dout=dout, cu_q=cu_q, cu_k=cu_k, B_k=B_k)


def _torch_out(L, q, kk, v, sm, dense):
    """Softmax attention of every (t, h) over its support, as torch ops."""
    sel, cu_q, cu_k, B_k = L["sel"], L["cu_q"], L["cu_k"], L["B_k"]
    T, H, d = q.shape
    G = kk.shape[1]
    Hg = H // G
    rows = []
    for b in range(len(cu_q) - 1):
        T_b, S_b = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        for i in range(T_b):
            t, pos = cu_q[b] + i, S_b - T_b + i
            heads = []
            for h in range(H):
                g = h // Hg
                chosen = {int(x) for x in sel[t, g] if x >= 0}
                mask = torch.tensor([dense or j // B_k in chosen for j in range(pos + 1)])
                s = sm * kk[cu_k[b]:cu_k[b] + pos + 1, g] @ q[t, h]
                s = torch.where(mask, s, torch.tensor(-float("inf"), dtype=s.dtype))
                heads.append(torch.softmax(s, 0) @ v[cu_k[b]:cu_k[b] + pos + 1, g])
            rows.append(torch.stack(heads))
    return torch.stack(rows)


@pytest.mark.parametrize("dense", [False, True])
def test_backward_matches_autograd(dense):
    L = _layer(1, S_lens=[17, 9, 1], T_lens=[17, 4, 1])
    sm = 0.6
    dq, dk, dv = B.main_branch_backward(L["q"], L["k"], L["v"], L["sel"], L["dout"], L["cu_q"], L["cu_k"], L["B_k"],
                                        sm, dense=dense)
    q = torch.from_numpy(L["q"]).requires_grad_(True)
    kk = torch.from_numpy(L["k"]).requires_grad_(True)
    v = torch.from_numpy(L["v"]).requires_grad_(True)
    out = _torch_out(L, q, kk, v, sm, dense)
    (out * torch.from_numpy(L["dout"])).sum().backward()
    np.testing.assert_allclose(dq, q.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, kk.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, v.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_matches_finite_differences():
    L = _layer(2, S_lens=[13, 6], T_lens=[13, 3])
    sm = 0.7
    dq, dk, dv = B.main_branch_backward(L["q"], L["k"], L["v"], L["sel"], L["dout"], L["cu_q"], L["cu_k"], L["B_k"], sm)
    T = L["cu_q"][-1]

    def loss(q, kk, v):
        o, _ = O.msa_forward_rows(q, kk, v, L["sel"], L["cu_q"], L["cu_k"], list(range(T)), L["B_k"], sm)
        return float((o * L["dout"]).sum())
    eps = 1e-6
    for name, arr, grad, idx in (("q", L["q"], dq, (5, 1, 2)), ("k", L["k"], dk, (3, 0, 1)),
                                 ("v", L["v"], dv, (14, 1, 3))):
        a, b = arr.copy(), arr.copy()
        a[idx] += eps
        b[idx] -= eps
        args_a = {"q": L["q"], "kk": L["k"], "v": L["v"]}
        args_b = dict(args_a)
        key = {"q": "q", "k": "kk", "v": "v"}[name]
        args_a[key], args_b[key] = a, b
        fd = (loss(**args_a) - loss(**args_b)) / (2 * eps)
        assert fd == pytest.approx(grad[idx], rel=1e-6, abs=1e-8), name


def test_one_token_support_closed_form():
    """The first query of a sequence (position 0) attends to one token only."""
    L = _layer(3, S_lens=[9], T_lens=[9], G=1, Hg=2)
    dq, dk, dv = B.main_branch_backward(L["q"], L["k"], L["v"], L["sel"], L["dout"], L["cu_q"], L["cu_k"], L["B_k"],
                                        0.5)
    assert np.allclose(dq[0], 0.0)
    # value 0 gets dO of query 0 (both heads) plus the shares of later queries
    only = B.main_branch_backward(L["q"][:1], L["k"][:1], L["v"][:1], L["sel"][:1], L["dout"][:1], [0, 1], [0, 1],
                                  L["B_k"], 0.5)
    np.testing.assert_allclose(only[2][0, 0], L["dout"][0].sum(axis=0), rtol=0, atol=1e-12)
    np.testing.assert_allclose(only[1][0, 0], 0.0, rtol=0, atol=1e-12)
