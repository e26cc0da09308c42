"""torch.autograd wrappers of the library's forward and backward calls, for
training with PyTorch.  Every step runs in the library's kernels; these
classes only route tensors and gradients.

* ``msa_attention(q, k, v, q_idx, k_idx, shape, seqs)`` -> (out, sel): the
  Index Branch selection and the Main Branch attention over it (prefill
  layout).  Backward: dq, dk, dv by msa_sparse_attn_backward; the selection is a
  top-k and gets no gradient, and neither do q_idx / k_idx through it.
* ``index_alignment_loss(q, k, q_idx, k_idx, sel, lse, shape, seqs, tau)`` ->
  the summed KL(P || Q) of the Index Branch against the Main Branch's attention
  on the support (pnsm.cn sec. 4: the teacher is held constant, so the
  gradient reaches q_idx and k_idx only).
"""
from __future__ import annotations

import torch

from block_sparse_long_exp_b200 import msa


class _MSAAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, q_idx, k_idx, shape, seqs):
        sel = msa.msa_index_topk(shape, seqs, q_idx, k_idx)
        out, lse = msa.msa_sparse_attn_prefill(shape, seqs, q, k, v, sel)
        ctx.save_for_backward(q, k, v, sel, out, lse)
        ctx.shape, ctx.seqs = shape, seqs
        ctx.mark_non_differentiable(sel)
        return out, sel

    @staticmethod
    def backward(ctx, d_out, d_sel):
        q, k, v, sel, out, lse = ctx.saved_tensors
        dq, dk, dv = msa.msa_sparse_attn_backward(ctx.shape, ctx.seqs, q, k, v, sel, out, lse,
                                                  d_out.to(torch.bfloat16).contiguous())
        return dq.to(q.dtype), dk.to(k.dtype), dv.to(v.dtype), None, None, None, None


class _IndexAlignmentLoss(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, q_idx, k_idx, sel, lse, shape, seqs, tau, dense):
        kl, lse_z = msa.msa_index_kl(shape, seqs, q, k, q_idx, k_idx, sel, lse, tau, dense=dense, want_lse_z=True)
        ctx.save_for_backward(q, k, q_idx, k_idx, sel if sel is not None else torch.empty(0), lse, lse_z)
        ctx.shape, ctx.seqs, ctx.tau, ctx.dense, ctx.has_sel = shape, seqs, tau, dense, sel is not None
        return kl.sum()

    @staticmethod
    def backward(ctx, g):
        q, k, q_idx, k_idx, sel, lse, lse_z = ctx.saved_tensors
        dq_idx, dk_idx = msa.msa_index_kl_backward(ctx.shape, ctx.seqs, q, k, q_idx, k_idx,
                                                   sel if ctx.has_sel else None, lse, lse_z, ctx.tau,
                                                   dense=ctx.dense)
        return (None, None, (g * dq_idx).to(q_idx.dtype), (g * dk_idx).to(k_idx.dtype), None, None, None, None,
                None, None)


def msa_attention(q, k, v, q_idx, k_idx, shape, seqs):
    """(out [T, H, d], sel [T, G, k]) with gradients for q, k and v."""
    return _MSAAttention.apply(q, k, v, q_idx, k_idx, shape, seqs)


def index_alignment_loss(q, k, q_idx, k_idx, sel, lse, shape, seqs, tau: float, dense: bool = False):
    """Summed KL(P || Q) over every (query, group); gradients for q_idx and
    k_idx only (the main-branch teacher is a constant of it).  lse: the
    forward's log-sum-exp over the same support (detached)."""
    return _IndexAlignmentLoss.apply(q.detach(), k.detach(), q_idx, k_idx, sel, lse.detach(), shape, seqs, tau,
                                     dense)
