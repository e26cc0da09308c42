"""The autograd wrappers on the GPU: a loss through msa_attention gives bf16
q, k and v the oracle's backward, and the index-alignment loss gives q_idx and
k_idx the oracle's KL gradient while q gets none.  Bound: 1e-2 of the largest
gradient, the kernels' own bounds (5e-3 backward, 2e-3 KL) plus the rounding
of every gradient to bf16 (2^-9 relative).  (Runs after the parity files.)"""
import numpy as np
import pytest
import torch

from oracle import index_kl as K
from oracle import main_backward as B
from test_gpu_parity import _custom, _f32, _inputs, _to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


def test_autograd_on_the_gpu(M):
    from block_sparse_long_exp_b200 import autograd as A
    w = _custom("autograd", 32, 2, 128, 64, 8, hot=0.05, seed=86)
    inp = _inputs(w, lengths=[900, 300], T_lens=[300, 300])
    shape, seqs, d = _to_dev(M, w, inp)
    q, k, v = (d[n].clone().requires_grad_(True) for n in ("q", "k", "v"))
    q_idx, k_idx = (d[n].clone().requires_grad_(True) for n in ("q_idx", "k_idx"))
    out, sel = A.msa_attention(q, k, v, q_idx, k_idx, shape, seqs)
    W = torch.randn(out.shape, generator=torch.Generator().manual_seed(3)).bfloat16().cuda()
    (out.float() * W.float()).sum().backward()
    torch.cuda.synchronize()
    assert q_idx.grad is None and k_idx.grad is None     # the selection is not differentiated
    sel_np = sel.cpu().numpy()
    want = B.main_branch_backward(_f32(inp["q"]), _f32(inp["k"]), _f32(inp["v"]), sel_np, _f32(W),
                                  inp["cu_q_host"], inp["cu_k_host"], w.B_k, w.sm_scale)
    for name, got, ref in zip(("dq", "dk", "dv"), (q.grad, k.grad, v.grad), want):
        assert got.dtype == torch.bfloat16, name
        np.testing.assert_allclose(_f32(got), ref, rtol=0, atol=1e-2 * np.abs(ref).max(), err_msg=name)
    # the index-alignment loss: gradients for the index query and keys only
    _, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
    q2 = d["q"].clone().requires_grad_(True)
    loss = A.index_alignment_loss(q2, d["k"], q_idx, k_idx, sel, lse, shape, seqs, tau=0.125)
    loss.backward()
    torch.cuda.synchronize()
    assert q2.grad is None
    _, dq_i, dk_i = K.index_kl_loss_and_grad(_f32(inp["q"]), _f32(inp["k"]), _f32(inp["q_idx"]), _f32(inp["k_idx"]),
                                             sel_np, inp["cu_q_host"], inp["cu_k_host"], w.B_k, w.sm_scale, 0.125)
    np.testing.assert_allclose(_f32(q_idx.grad), dq_i, rtol=0, atol=1e-2 * np.abs(dq_i).max())
    np.testing.assert_allclose(_f32(k_idx.grad), dk_i, rtol=0, atol=1e-2 * np.abs(dk_i).max())
