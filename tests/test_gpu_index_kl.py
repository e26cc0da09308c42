"""The index-alignment target on the GPU (msa_index_kl and its gradient,
msa_index_kl_backward) against the fp64 oracle (oracle/index_kl.py) on every
row of a ragged varlen layer whose
queries are the last T_b tokens: the sparse support with the selection the
library computed, and the dense (warmup) support.  The log-sum-exps come from
the oracle (the kernel alone is compared) and then from the library's own
prefill and dense calls (the chain a training step would run).  A selected
block past the query's block is reported, not read.  (Runs after the parity
files.)"""
import numpy as np
import pytest
import torch

from oracle import index_kl as K
from oracle import msa_oracle as O
from test_gpu_parity import _custom, _f32, _inputs, _to_dev

pytestmark = pytest.mark.gpu

TAU = 0.125


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


def _case(M):
    w = _custom("index_kl", 64, 4, 128, 64, 16, hot=0.05, seed=97)
    inp = _inputs(w, lengths=[2100, 129, 1300], T_lens=[700, 129, 400])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    return w, inp, shape, seqs, d, sel


def _host(inp):
    return {k: _f32(inp[k]).astype(np.float64) for k in ("q", "k", "v", "q_idx", "k_idx")}


@pytest.mark.parametrize("dense", [False, True])
def test_index_kl_matches_the_oracle(M, dense):
    w, inp, shape, seqs, d, sel = _case(M)
    h = _host(inp)
    cu_q, cu_k = inp["cu_q_host"], inp["cu_k_host"]
    T = cu_q[-1]
    rows = list(range(T))
    sel_np = sel.cpu().numpy()
    use = np.tile(np.arange(64, dtype=np.int32)[None, None, :], (T, w.G, 1)) if dense else sel_np
    _, lse_ref = O.msa_forward_rows(h["q"], h["k"], h["v"], use, cu_q, cu_k, rows, w.B_k, w.sm_scale)
    want = K.index_kl_rows(h["q"], h["k"], h["q_idx"], h["k_idx"], sel_np, cu_q, cu_k, rows, w.B_k, w.sm_scale,
                           TAU, dense=dense)
    lse_dev = torch.from_numpy(lse_ref.astype(np.float32)).cuda()
    s_arg = None if dense else sel
    kl, lse_z = M.msa_index_kl(shape, seqs, d["q"], d["k"], d["q_idx"], d["k_idx"], s_arg, lse_dev, TAU,
                               dense=dense, want_lse_z=True)
    dq, dk = M.msa_index_kl_backward(shape, seqs, d["q"], d["k"], d["q_idx"], d["k_idx"], s_arg, lse_dev, lse_z,
                                     TAU, dense=dense)
    torch.cuda.synchronize()
    got = kl.cpu().numpy()
    assert np.all(np.isfinite(got)) and np.all(want > -1e-9)
    np.testing.assert_allclose(got, want, rtol=1e-3, atol=1e-3)
    # gradient with respect to the index query and keys, the teacher held constant
    _, want_dq, want_dk = K.index_kl_loss_and_grad(h["q"], h["k"], h["q_idx"], h["k_idx"], sel_np, cu_q, cu_k,
                                                   w.B_k, w.sm_scale, TAU, dense=dense)
    np.testing.assert_allclose(dq.cpu().numpy(), want_dq, rtol=0, atol=2e-3 * np.abs(want_dq).max())
    np.testing.assert_allclose(dk.cpu().numpy(), want_dk, rtol=0, atol=2e-3 * np.abs(want_dk).max())
    # the same with the library's own log-sum-exps
    if dense:
        _, lse_lib = M.msa_dense_attn(shape, seqs, d["q"], d["k"], d["v"], want_lse=True)
    else:
        _, lse_lib = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
    kl2 = M.msa_index_kl(shape, seqs, d["q"], d["k"], d["q_idx"], d["k_idx"], None if dense else sel, lse_lib, TAU,
                         dense=dense)
    torch.cuda.synchronize()
    np.testing.assert_allclose(kl2.cpu().numpy(), want, rtol=5e-3, atol=5e-3)


# The tensor-core target and gradient over (H, G, d, d_idx): 4 and 8 heads per
# group (8 tile rows per query), index rows of 64 and 256 bytes (their two
# swizzle widths and two boxes per row), and the shape whose key and
# index-key tiles leave room for one key stage
@pytest.mark.parametrize("H,G,d,d_idx", [(16, 4, 64, 32), (32, 4, 128, 128), (16, 1, 64, 128), (16, 2, 128, 64)])
def test_index_kl_tensor_core_shapes(M, H, G, d, d_idx):
    w = _custom("index_kl_shapes", H, G, d, d_idx, 8, hot=0.05, seed=31 + H + d_idx)
    inp = _inputs(w, lengths=[1500, 300], T_lens=[600, 300])
    shape, seqs, dv = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, dv["q_idx"], dv["k_idx"])
    h = _host(inp)
    cu_q, cu_k = inp["cu_q_host"], inp["cu_k_host"]
    rows = list(range(cu_q[-1]))
    sel_np = sel.cpu().numpy()
    _, lse_ref = O.msa_forward_rows(h["q"], h["k"], h["v"], sel_np, cu_q, cu_k, rows, w.B_k, w.sm_scale)
    want = K.index_kl_rows(h["q"], h["k"], h["q_idx"], h["k_idx"], sel_np, cu_q, cu_k, rows, w.B_k, w.sm_scale,
                           TAU)
    lse_dev = torch.from_numpy(lse_ref.astype(np.float32)).cuda()
    kl, lse_z = M.msa_index_kl(shape, seqs, dv["q"], dv["k"], dv["q_idx"], dv["k_idx"], sel, lse_dev, TAU,
                               want_lse_z=True)
    dq, dk = M.msa_index_kl_backward(shape, seqs, dv["q"], dv["k"], dv["q_idx"], dv["k_idx"], sel, lse_dev, lse_z,
                                     TAU)
    torch.cuda.synchronize()
    got = kl.cpu().numpy()
    assert np.all(np.isfinite(got)) and np.all(np.isfinite(lse_z.cpu().numpy()))
    np.testing.assert_allclose(got, want, rtol=1e-3, atol=1e-3)
    _, want_dq, want_dk = K.index_kl_loss_and_grad(h["q"], h["k"], h["q_idx"], h["k_idx"], sel_np, cu_q, cu_k,
                                                   w.B_k, w.sm_scale, TAU)
    np.testing.assert_allclose(dq.cpu().numpy(), want_dq, rtol=0, atol=2e-3 * np.abs(want_dq).max())
    np.testing.assert_allclose(dk.cpu().numpy(), want_dk, rtol=0, atol=2e-3 * np.abs(want_dk).max())


def test_index_kl_bad_block_is_reported(M):
    w, inp, shape, seqs, d, sel = _case(M)
    bad = sel.clone()
    row = inp["cu_q_host"][1]                 # sequence 1's first query sits at position 0
    bad[row, 1, 0] = 5                        # block 5 is in its future
    lse = torch.zeros(seqs.total_q, w.H, device="cuda")
    with pytest.raises(M.MsaError, match="DEVICE_CHECK"):
        M.msa_index_kl(shape, seqs, d["q"], d["k"], d["q_idx"], d["k_idx"], bad, lse, TAU)
    torch.cuda.synchronize()                  # the context is still usable
    M.msa_index_kl(shape, seqs, d["q"], d["k"], d["q_idx"], d["k_idx"], sel, lse, TAU)
