"""The Main Branch backward on the GPU (msa_sparse_attn_backward) against the
fp64 oracle (oracle/main_backward.py) on a ragged varlen layer whose queries
are the last T_b tokens: the sparse support with the library's selection and
forward outputs, and the dense support with the dense call's outputs, as a
training step would chain them.  A selected block past the query's block is
reported, not read.  (Runs after the parity files.)"""
import numpy as np
import pytest
import torch

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


def _case(M):
    # 16 heads per group and d = 128: every thread keeps its full 16 dq outputs
    w = _custom("attn_bwd", 32, 2, 128, 64, 8, hot=0.05, seed=89)
    inp = _inputs(w, lengths=[1500, 129, 700], T_lens=[250, 129, 200])
    shape, seqs, d = _to_dev(M, w, inp)
    gen = torch.Generator().manual_seed(90)
    dout = torch.randn(inp["q"].shape, generator=gen).bfloat16()
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    return w, inp, shape, seqs, d, sel, dout


@pytest.mark.parametrize("dense", [False, True])
def test_backward_matches_the_oracle(M, dense):
    w, inp, shape, seqs, d, sel, dout = _case(M)
    if dense:
        out, lse = M.msa_dense_attn(shape, seqs, d["q"], d["k"], d["v"], want_lse=True)
    else:
        out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
    dq, dk, dv = M.msa_sparse_attn_backward(shape, seqs, d["q"], d["k"], d["v"], None if dense else sel, out, lse,
                                            dout.cuda(), dense=dense)
    torch.cuda.synchronize()
    want = B.main_branch_backward(_f32(inp["q"]), _f32(inp["k"]), _f32(inp["v"]), sel.cpu().numpy(), _f32(dout),
                                  inp["cu_q_host"], inp["cu_k_host"], w.B_k, w.sm_scale, dense=dense)
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
        g = got.cpu().numpy()
        assert np.all(np.isfinite(g)), name
        np.testing.assert_allclose(g, ref, rtol=0, atol=5e-3 * np.abs(ref).max(), err_msg=name)


# The tensor-core form over (H, G, d): 4, 8 and 16 heads per group (8 or 16
# tile rows per query) and d = 64 (two key stages and two query slots in
# shared memory) and 128 (one of each)
@pytest.mark.parametrize("H,G,d", [(16, 4, 64), (32, 4, 128), (16, 1, 64), (32, 2, 64)])
def test_backward_tensor_core_shapes(M, H, G, d):
    w = _custom("attn_bwd_shapes", H, G, d, 64, 8, hot=0.05, seed=61 + H + d)
    inp = _inputs(w, lengths=[1400, 300], T_lens=[500, 300])
    shape, seqs, dv_ = _to_dev(M, w, inp)
    gen = torch.Generator().manual_seed(62 + d)
    dout = torch.randn(inp["q"].shape, generator=gen).bfloat16()
    sel = M.msa_index_topk(shape, seqs, dv_["q_idx"], dv_["k_idx"])
    out, lse = M.msa_sparse_attn_prefill(shape, seqs, dv_["q"], dv_["k"], dv_["v"], sel)
    dq, dk, dv = M.msa_sparse_attn_backward(shape, seqs, dv_["q"], dv_["k"], dv_["v"], sel, out, lse, dout.cuda())
    torch.cuda.synchronize()
    want = B.main_branch_backward(_f32(inp["q"]), _f32(inp["k"]), _f32(inp["v"]), sel.cpu().numpy(), _f32(dout),
                                  inp["cu_q_host"], inp["cu_k_host"], w.B_k, w.sm_scale)
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
        g = got.cpu().numpy()
        assert np.all(np.isfinite(g)), name
        np.testing.assert_allclose(g, ref, rtol=0, atol=5e-3 * np.abs(ref).max(), err_msg=name)


def test_backward_bad_block_is_reported(M):
    w, inp, shape, seqs, d, sel, dout = _case(M)
    out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
    bad = sel.clone()
    row = inp["cu_q_host"][1]                 # sequence 1's first query sits at position 0
    bad[row, 1, 0] = 7                        # block 7 is in its future
    with pytest.raises(M.MsaError, match="DEVICE_CHECK"):
        M.msa_sparse_attn_backward(shape, seqs, d["q"], d["k"], d["v"], bad, out, lse, dout.cuda())
    torch.cuda.synchronize()                  # the context is still usable
    M.msa_sparse_attn_backward(shape, seqs, d["q"], d["k"], d["v"], sel, out, lse, dout.cuda())
