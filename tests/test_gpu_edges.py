"""Edge cases of the method and of the inputs, each against the oracle:
k = 1 (the local block alone), a sequence with no queries inside a batch, a
call with no queries at all, a one-token sequence, lengths at and around
block boundaries, decode with k = 1.  Every path of the prefill split
(query tiles on and off) is run."""
import numpy as np
import pytest
import torch

from test_gpu_parity import _check_out, _custom, _inputs, _oracle_out, _oracle_sel, _to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


def _prefill(M, w, inp, theta):
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    prev = M.msa_set_tile_threshold(theta)
    try:
        out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
    finally:
        M.msa_set_tile_threshold(prev)
    torch.cuda.synchronize()
    return sel, out, lse


@pytest.mark.parametrize("theta", [0, -1])
def test_k1_local_block_only(M, theta):
    w = _custom("k1", 64, 4, 128, 64, 1, seed=71)
    inp = _inputs(w, lengths=[1000, 129])
    sel, out, lse = _prefill(M, w, inp, theta)
    ref = _oracle_sel(w, inp)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref)
    t = np.arange(inp["cu_q_host"][-1])
    pos = np.where(t < 1000, t, t - 1000)
    assert np.all(sel.cpu().numpy()[:, :, 0] == (pos // 128)[:, None])   # only the own block
    o_ref, l_ref = _oracle_out(w, inp, ref)
    _check_out(out, lse, o_ref, l_ref)


@pytest.mark.parametrize("theta", [0, -1])
def test_sequence_without_queries(M, theta):
    """A sequence whose query range is empty, between two that have queries."""
    w = _custom("emptyq", 64, 4, 128, 64, 16, hot=0.05, seed=72)
    inp = _inputs(w, lengths=[2000, 1500, 900], T_lens=[700, 0, 900])
    sel, out, lse = _prefill(M, w, inp, theta)
    ref = _oracle_sel(w, inp)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref)
    o_ref, l_ref = _oracle_out(w, inp, ref)
    _check_out(out, lse, o_ref, l_ref)


def test_no_queries_at_all(M):
    """total_q = 0: every call succeeds and writes nothing."""
    w = _custom("noq", 64, 4, 128, 64, 16, seed=73)
    inp = _inputs(w, lengths=[500, 300], T_lens=[0, 0])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    assert sel.numel() == 0
    out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
    assert out.numel() == 0 and lse.numel() == 0
    out2, _ = M.msa_dense_attn(shape, seqs, d["q"], d["k"], d["v"])
    assert out2.numel() == 0


@pytest.mark.parametrize("theta", [0, 1])
def test_one_token_and_block_boundaries(M, theta):
    """Lengths 1, 127, 128, 129, 255, 256, 257: partial, exact and just-over blocks."""
    w = _custom("bounds", 64, 4, 128, 64, 2, hot=0.0, seed=74)
    inp = _inputs(w, lengths=[1, 127, 128, 129, 255, 256, 257])
    sel, out, lse = _prefill(M, w, inp, theta)
    ref = _oracle_sel(w, inp)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref)
    o_ref, l_ref = _oracle_out(w, inp, ref)
    _check_out(out, lse, o_ref, l_ref)


def test_decode_k1_and_short_caches(M):
    w = _custom("deck1", 64, 4, 128, 64, 1, seed=75, kind="decode")
    inp = _inputs(w, lengths=[1, 128, 129, 4000])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    ref = _oracle_sel(w, inp)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref)
    out, lse = M.msa_sparse_attn_decode(shape, seqs, d["q"], d["k"], d["v"], sel)
    o_ref, l_ref = _oracle_out(w, inp, ref)
    _check_out(out, lse, o_ref, l_ref)
