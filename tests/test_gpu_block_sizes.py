"""Block sizes B_k = 32 and 64 on the main path (the pages' block-size ablation,
pnsm.cn explainer sec. 8: PPL close across 32 / 64 / 128, larger blocks trading
for kernel efficiency).  The index kernels max-pool each 128-key tile into
128 / B_k block scores; the attention kernels read a block's 128-row K/V tile
and attend its first B_k keys.  Selections must equal the fp64 oracle's bit
for bit; outputs within max-abs 2e-2 and mean-relative 5e-3."""
import numpy as np
import pytest
import torch

from block_sparse_long_exp_b200 import workloads as W
from test_gpu_parity import _check_out, _inputs, _oracle_out, _oracle_sel, _to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


def _w(name, B_k, k, H=64, G=4, d=128, d_idx=64, hot=0.05, seed=61, kind="prefill"):
    return W.Workload(name, kind, H=H, G=G, d=d, d_idx=d_idx, B_k=B_k, k=k, seed=seed, hot_frac=hot)


@pytest.mark.parametrize("B_k,k", [(64, 16), (64, 32), (32, 16), (32, 32), (32, 8)])
def test_prefill_index_and_attention(M, B_k, k):
    """Ragged varlen prefill with hot blocks: selection exact, outputs within
    tolerance, query tiles on (automatic threshold) and off (all KV-outer)."""
    w = _w("bk", B_k, k, seed=61 + B_k + k)
    inp = _inputs(w, lengths=[2600, 130, 1901, 63])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    ref_sel = _oracle_sel(w, inp)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref_sel)
    o_ref, lse_ref = _oracle_out(w, inp, ref_sel)
    for theta in (-1, 0):
        prev = M.msa_set_tile_threshold(theta)
        try:
            out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
        finally:
            M.msa_set_tile_threshold(prev)
        _check_out(out, lse, o_ref, lse_ref)


@pytest.mark.parametrize("B_k", [32, 64])
def test_chunked_prefill_last_tokens_and_passes(M, B_k):
    """Queries are the last T_b tokens of their sequence (chunked prefill), in
    passes of 700 rows, with small heads (H/G = 8, d = 64, d_idx = 32)."""
    w = _w("bkc", B_k, 12, H=16, G=2, d=64, d_idx=32, seed=70 + B_k)
    inp = _inputs(w, lengths=[3000, 1300], T_lens=[900, 1300])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    ref_sel = _oracle_sel(w, inp)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref_sel)
    out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel, q_chunk=700)
    o_ref, lse_ref = _oracle_out(w, inp, ref_sel)
    _check_out(out, lse, o_ref, lse_ref)


@pytest.mark.parametrize("B_k", [32, 64])
def test_decode(M, B_k):
    """One query per sequence (lengths around block and tile edges)."""
    w = _w("bkd", B_k, 16, seed=80 + B_k, hot=0.02, kind="decode")
    inp = _inputs(w, lengths=[1, 31, 32, 33, 127, 129, 5000, 2049])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    ref_sel = _oracle_sel(w, inp)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref_sel)
    out, lse = M.msa_sparse_attn_decode(shape, seqs, d["q"], d["k"], d["v"], sel)
    o_ref, lse_ref = _oracle_out(w, inp, ref_sel)
    _check_out(out, lse, o_ref, lse_ref)


@pytest.mark.parametrize("B_k", [32, 64])
def test_every_block_selected_is_dense(M, B_k):
    """k >= the number of causal blocks: every block selected, equal to dense
    causal GQA (the oracle's pinned special case)."""
    w = _w("bkdense", B_k, 32, H=16, G=2, d=64, d_idx=32, hot=0.0, seed=90 + B_k)
    inp = _inputs(w, lengths=[B_k * 32 - 5])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    s = sel.cpu().numpy()
    for t in (0, B_k - 1, B_k, B_k * 32 - 6):
        nb = t // B_k + 1
        assert s[t, 0, :nb].tolist() == list(range(nb)) and np.all(s[t, 0, nb:] == -1)
    out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
    o_ref, lse_ref = _oracle_out(w, inp, s)
    _check_out(out, lse, o_ref, lse_ref)
