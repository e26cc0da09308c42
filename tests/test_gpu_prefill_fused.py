"""GPU tests of msa_prefill, the one-call MSA layer (index top-k, then the
main branch, in passes of q_chunk query rows, the combine of a pass on a
second stream while the next pass's index top-k runs): its selection and
outputs must equal, bit for bit, those of msa_index_topk followed by
msa_sparse_attn_prefill with the same q_chunk, for every pass size (multiples
of the 128-query index tile or not), ragged batches, queries that are the last
tokens of longer sequences, block sizes 64 and 128, and the overlap on or off.
One case is also checked against the fp64 oracle directly."""

import pytest
import torch

from test_gpu_parity import _check_out, _custom, _inputs, _oracle_out, _oracle_sel, _to_dev
from block_sparse_long_exp_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


def _separate(M, shape, seqs, d, q_chunk):
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel, q_chunk=q_chunk)
    return sel, out, lse


def _fused(M, shape, seqs, d, q_chunk, overlap):
    prev = M.msa_set_prefill_overlap(overlap)
    try:
        return M.msa_prefill(shape, seqs, d["q"], d["k"], d["v"], d["q_idx"], d["k_idx"], q_chunk=q_chunk)
    finally:
        M.msa_set_prefill_overlap(prev)


def _assert_same(got, ref):
    for g, r in zip(got, ref):
        assert g.shape == r.shape and g.dtype == r.dtype
        assert torch.equal(g, r)


@pytest.mark.parametrize("q_chunk,overlap", [(0, -1), (700, -1), (700, 32), (1000, 16), (128, 48), (2048, 74),
                                             (3000, 24)])
def test_fused_equals_separate_calls(M, q_chunk, overlap):
    w = _custom("fused", 64, 4, 128, 64, 16, hot=0.05, seed=31)
    inp = _inputs(w, lengths=[2600, 130, 1901, 777])
    shape, seqs, d = _to_dev(M, w, inp)
    ref = _separate(M, shape, seqs, d, q_chunk)
    _assert_same(_fused(M, shape, seqs, d, q_chunk, overlap), ref)


def test_fused_queries_are_last_tokens_and_block_64(M):
    w = W.Workload("fused64", "prefill", H=64, G=4, d=128, d_idx=64, B_k=64, k=16, seed=32, hot_frac=0.05)
    inp = _inputs(w, lengths=[2000, 1300, 513], T_lens=[300, 1300, 200])
    shape, seqs, d = _to_dev(M, w, inp)
    for q_chunk in (0, 257):
        ref = _separate(M, shape, seqs, d, q_chunk)
        _assert_same(_fused(M, shape, seqs, d, q_chunk, -1), ref)


def test_fused_against_the_oracle(M):
    w = _custom("fused_oracle", 64, 4, 128, 64, 16, hot=0.05, seed=33)
    inp = _inputs(w, lengths=[1500, 900])
    shape, seqs, d = _to_dev(M, w, inp)
    sel, out, lse = _fused(M, shape, seqs, d, 640, -1)
    ref_sel = _oracle_sel(w, inp)
    assert (sel.cpu().numpy() == ref_sel).all()
    o_ref, lse_ref = _oracle_out(w, inp, ref_sel)
    _check_out(out, lse, o_ref, lse_ref)


def test_fused_full_size_in_four_passes(M):
    """The 128K-token layer with 2% hot blocks in four passes of 32768 rows,
    with and without the overlap, against the separate calls."""
    w = W.WORKLOADS["prefill_n131072_hot2"]
    inp = W.make_inputs(w, "cuda")
    shape = M.make_shape(w.H, w.G, w.d, w.d_idx, w.k, B_k=w.B_k)
    seqs = M.make_varlen(inp["cu_q"], inp["cu_k"], inp["cu_q_host"], inp["cu_k_host"])
    ref = _separate(M, shape, seqs, inp, 32768)
    for overlap in (0, 32):
        _assert_same(_fused(M, shape, seqs, inp, 32768, overlap), ref)
    del ref, inp
    torch.cuda.empty_cache()
