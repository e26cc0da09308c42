"""The autograd wrappers (block_sparse_long_exp_b200/autograd.py) route the
library's gradients to the right tensors: with the five library calls replaced
by the pinned fp64 oracles (no GPU here), a loss through msa_attention gives
q, k and v exactly the oracle's backward, and the index-alignment loss gives
q_idx and k_idx the oracle's KL gradient and leaves q, k untouched (the
teacher is held constant)."""
import math

import numpy as np
import pytest
import torch

from block_sparse_long_exp_b200 import autograd as A
from block_sparse_long_exp_b200 import msa
from oracle import index_kl as K
from oracle import main_backward as B
from oracle import msa_oracle as O

B_k = 4


class _Seqs:
    def __init__(self, cu_q, cu_k):
        self.cu_q, self.cu_k = cu_q, cu_k


def _np(t):
    return t.detach().double().numpy()


@pytest.fixture
def fakes(monkeypatch):
    def topk(shape, seqs, q_idx, k_idx):
        return torch.from_numpy(O.index_topk(_np(q_idx), _np(k_idx), seqs.cu_q, seqs.cu_k, shape.k, B_k))

    def prefill(shape, seqs, q, k, v, sel):
        T = seqs.cu_q[-1]
        o, lse = O.msa_forward_rows(_np(q), _np(k), _np(v), sel.numpy(), seqs.cu_q, seqs.cu_k, list(range(T)), B_k,
                                    shape.sm_scale)
        return torch.from_numpy(o).to(q.dtype), torch.from_numpy(lse).float()

    def backward(shape, seqs, q, k, v, sel, out, lse, dout, dense=False):
        r = B.main_branch_backward(_np(q), _np(k), _np(v), sel.numpy(), _np(dout), seqs.cu_q, seqs.cu_k, B_k,
                                   shape.sm_scale, dense=dense)
        return tuple(torch.from_numpy(x).float() for x in r)

    def kl(shape, seqs, q, k, q_idx, k_idx, sel, lse, tau, dense=False, want_lse_z=False):
        T = seqs.cu_q[-1]
        v = K.index_kl_rows(_np(q), _np(k), _np(q_idx), _np(k_idx), sel.numpy(), seqs.cu_q, seqs.cu_k,
                            list(range(T)), B_k, shape.sm_scale, tau, dense=dense)
        return torch.from_numpy(v).float(), torch.zeros(T, shape.G)

    def kl_backward(shape, seqs, q, k, q_idx, k_idx, sel, lse, lse_z, tau, dense=False):
        _, dq, dk = K.index_kl_loss_and_grad(_np(q), _np(k), _np(q_idx), _np(k_idx), sel.numpy(), seqs.cu_q,
                                             seqs.cu_k, B_k, shape.sm_scale, tau, dense=dense)
        return torch.from_numpy(dq).float(), torch.from_numpy(dk).float()

    for name, fn in (("msa_index_topk", topk), ("msa_sparse_attn_prefill", prefill),
                     ("msa_sparse_attn_backward", backward), ("msa_index_kl", kl),
                     ("msa_index_kl_backward", kl_backward)):
        monkeypatch.setattr(msa, name, fn)


def _layer():
    rng = np.random.default_rng(8)
    H, G, d, d_idx = 4, 2, 8, 4
    S_lens, T_lens = [19, 10], [19, 6]
    cu_k = np.concatenate([[0], np.cumsum(S_lens)]).tolist()
    cu_q = np.concatenate([[0], np.cumsum(T_lens)]).tolist()
    T, S = cu_q[-1], cu_k[-1]
    mk = lambda *s: torch.from_numpy(rng.standard_normal(s)).to(torch.float64)  # noqa: E731
    shape = msa.make_shape(H, G, d, d_idx, 2, B_k=B_k)
    return shape, _Seqs(cu_q, cu_k), mk(T, H, d), mk(S, G, d), mk(S, G, d), mk(T, G, d_idx), mk(S, d_idx)


def test_attention_gradients_are_the_backward(fakes):
    shape, seqs, q, k, v, q_idx, k_idx = _layer()
    for t in (q, k, v):
        t.requires_grad_(True)
    out, sel = A.msa_attention(q, k, v, q_idx, k_idx, shape, seqs)
    assert not sel.requires_grad
    W = torch.randn(out.shape, dtype=torch.float64).bfloat16().double()   # dout exactly representable in bf16
    (out * W).sum().backward()
    want = B.main_branch_backward(_np(q), _np(k), _np(v), sel.numpy(), _np(W), seqs.cu_q, seqs.cu_k, B_k,
                                  shape.sm_scale)
    for got, ref in zip((q.grad, k.grad, v.grad), want):
        np.testing.assert_allclose(got.numpy(), ref, rtol=1e-6, atol=1e-6)


def test_index_alignment_gradients_reach_the_index_only(fakes):
    shape, seqs, q, k, v, q_idx, k_idx = _layer()
    q.requires_grad_(True)
    q_idx.requires_grad_(True)
    k_idx.requires_grad_(True)
    sel = torch.from_numpy(O.index_topk(_np(q_idx), _np(k_idx), seqs.cu_q, seqs.cu_k, shape.k, B_k))
    lse = torch.zeros(q.shape[0], shape.H)
    loss = A.index_alignment_loss(q, k, q_idx, k_idx, sel, lse, shape, seqs, tau=0.5)
    (3.0 * loss).backward()
    _, dq, dk = K.index_kl_loss_and_grad(_np(q), _np(k), _np(q_idx), _np(k_idx), sel.numpy(), seqs.cu_q, seqs.cu_k,
                                         B_k, shape.sm_scale, 0.5)
    np.testing.assert_allclose(q_idx.grad.numpy(), 3.0 * dq, rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(k_idx.grad.numpy(), 3.0 * dk, rtol=1e-6, atol=1e-6)
    assert q.grad is None                       # the teacher side gets no gradient
    assert math.isfinite(loss.item())
