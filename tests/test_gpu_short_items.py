"""The tensor-core training kernels on work items of one tile: many short
sequences whose KV-outer lists hold a few queries each, so that a warpgroup
often takes none of an item's tiles and the item ring runs ahead of the key
stages (the condition under which a stage could be released before every
reader of it is done).  The KL target, its gradient and the Main Branch
backward against the fp64 oracle, three launches each: the KL target writes
every partial once and merges them in a fixed order, so it must repeat bit for
bit; the gradients (added with reductions) within the parity tests' bounds
every time.  (Runs after the other training files.)"""
import numpy as np
import pytest
import torch

from oracle import index_kl as K
from oracle import main_backward as B
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


def _short_case(M, H, G, d, d_idx, seed):
    w = _custom("short_items", H, G, d, d_idx, 4, hot=0.0, seed=seed)
    rng = np.random.default_rng(seed)
    lengths = [int(x) for x in rng.integers(40, 420, size=24)]
    T_lens = [int(min(L, x)) for L, x in zip(lengths, rng.integers(1, 24, size=24))]
    inp = _inputs(w, lengths=lengths, T_lens=T_lens)
    shape, seqs, dv = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, dv["q_idx"], dv["k_idx"])
    return w, inp, shape, seqs, dv, sel


# 8 tile rows per query with one key stage (d = d_idx = 128), and 16 rows per
# query with two (d = d_idx = 64)
@pytest.mark.parametrize("H,G,d,d_idx", [(32, 4, 128, 128), (32, 2, 64, 64)])
def test_training_kernels_on_single_tile_items(M, H, G, d, d_idx):
    w, inp, shape, seqs, dv, sel = _short_case(M, H, G, d, d_idx, 71 + H + d_idx)
    h = {n: _f32(inp[n]).astype(np.float64) for n in ("q", "k", "v", "q_idx", "k_idx")}
    cu_q, cu_k = inp["cu_q_host"], inp["cu_k_host"]
    T = cu_q[-1]
    rows = list(range(T))
    sel_np = sel.cpu().numpy()
    _, lse_ref = O.msa_forward_rows(h["q"], h["k"], h["v"], sel_np, cu_q, cu_k, rows, w.B_k, w.sm_scale)
    lse_dev = torch.from_numpy(lse_ref.astype(np.float32)).cuda()
    want_kl = K.index_kl_rows(h["q"], h["k"], h["q_idx"], h["k_idx"], sel_np, cu_q, cu_k, rows, w.B_k, w.sm_scale,
                              TAU)
    _, want_dq_idx, want_dk_idx = K.index_kl_loss_and_grad(h["q"], h["k"], h["q_idx"], h["k_idx"], sel_np, cu_q,
                                                           cu_k, w.B_k, w.sm_scale, TAU)
    out, lse = M.msa_sparse_attn_prefill(shape, seqs, dv["q"], dv["k"], dv["v"], sel)
    gen = torch.Generator().manual_seed(5 + d)
    dout = torch.randn(inp["q"].shape, generator=gen).bfloat16()
    want_bwd = B.main_branch_backward(h["q"], h["k"], h["v"], sel_np, _f32(dout), cu_q, cu_k, w.B_k, w.sm_scale)
    first = None
    for _ in range(3):
        kl, lse_z = M.msa_index_kl(shape, seqs, dv["q"], dv["k"], dv["q_idx"], dv["k_idx"], sel, lse_dev, TAU,
                                   want_lse_z=True)
        dq_idx, dk_idx = M.msa_index_kl_backward(shape, seqs, dv["q"], dv["k"], dv["q_idx"], dv["k_idx"], sel,
                                                 lse_dev, lse_z, TAU)
        dq, dk, dvv = M.msa_sparse_attn_backward(shape, seqs, dv["q"], dv["k"], dv["v"], sel, out, lse,
                                                 dout.cuda())
        torch.cuda.synchronize()
        got = kl.cpu().numpy()
        if first is None:
            first = got.copy()
        assert np.array_equal(got, first)
        np.testing.assert_allclose(got, want_kl, rtol=1e-3, atol=1e-3)
        for name, a, ref in (("dq_idx", dq_idx, want_dq_idx), ("dk_idx", dk_idx, want_dk_idx)):
            np.testing.assert_allclose(a.cpu().numpy(), ref, rtol=0, atol=2e-3 * np.abs(ref).max(), err_msg=name)
        for name, a, ref in zip(("dq", "dk", "dv"), (dq, dk, dvv), want_bwd):
            np.testing.assert_allclose(a.cpu().numpy(), ref, rtol=0, atol=5e-3 * np.abs(ref).max(), err_msg=name)
