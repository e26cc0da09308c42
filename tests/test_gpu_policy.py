"""The scored selection policies on the GPU (msa_index_topk_policy): with no
sink and a one-block window its selection equals msa_index_topk's (the tensor
core kernel) bit for bit; with forced sinks and local windows it equals the
selection-policy oracle on every row; and the main branch attends a policy's
selection like any other.  (Runs after the parity files.)"""
import numpy as np
import pytest
import torch

from oracle import selection_policies as P
from test_gpu_parity import _check_out, _custom, _f32, _inputs, _oracle_out, _to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


def _case(M):
    w = _custom("policy", 64, 4, 128, 64, 16, hot=0.05, seed=85)
    inp = _inputs(w, lengths=[3000, 129, 2200], T_lens=[600, 129, 500])
    return (w, inp) + _to_dev(M, w, inp)


def test_final_rule_equals_the_tensor_core_kernel(M):
    w, inp, shape, seqs, d = _case(M)
    a = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    b = M.msa_index_topk_policy(shape, seqs, d["q_idx"], d["k_idx"], n_sink=0, n_local=1)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("n_sink,n_local", [(1, 1), (2, 3), (1, 15)])
def test_policies_match_the_oracle_and_attend(M, n_sink, n_local):
    w, inp, shape, seqs, d = _case(M)
    sel = M.msa_index_topk_policy(shape, seqs, d["q_idx"], d["k_idx"], n_sink=n_sink, n_local=n_local)
    torch.cuda.synchronize()
    ref = P.index_topk_policy(_f32(inp["q_idx"]), _f32(inp["k_idx"]), inp["cu_q_host"], inp["cu_k_host"], w.k, w.B_k,
                              n_sink, n_local)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref)
    if (n_sink, n_local) == (1, 1):
        out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
        torch.cuda.synchronize()
        o_ref, l_ref = _oracle_out(w, inp, ref)
        _check_out(out, lse, o_ref, l_ref)
