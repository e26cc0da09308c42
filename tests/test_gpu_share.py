"""The selection's share of the dense attention weight on the GPU
(msa_selected_share over the prefill and dense calls' log-sum-exps) against
the oracle's direct definition (oracle/index_kl.py: the dense causal softmax
summed over the selected tokens) on every (query, head) of a ragged layer.
(Runs after the parity files.)"""
import numpy as np
import pytest
import torch

from oracle import index_kl as K
from test_gpu_parity import _custom, _f32, _inputs, _to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


def test_selected_share_matches_the_definition(M):
    w = _custom("share", 32, 2, 128, 64, 8, hot=0.05, seed=87)
    inp = _inputs(w, lengths=[2100, 300, 1000], T_lens=[500, 300, 250])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    _, lse_sel = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
    _, lse_all = M.msa_dense_attn(shape, seqs, d["q"], d["k"], d["v"], want_lse=True)
    share = M.msa_selected_share(lse_sel, lse_all)
    torch.cuda.synchronize()
    T = inp["cu_q_host"][-1]
    want = K.selected_attention_mass(_f32(inp["q"]), _f32(inp["k"]), sel.cpu().numpy(), inp["cu_q_host"],
                                     inp["cu_k_host"], list(range(T)), w.B_k, w.sm_scale)
    got = share.cpu().numpy()
    np.testing.assert_allclose(got, want, rtol=0, atol=2e-3)
    assert np.all(got <= 1.0 + 2e-3)
    # sequence 1 (300 tokens, 3 blocks <= k) selects every causal block: all of the weight
    np.testing.assert_allclose(got[500:800], 1.0, rtol=0, atol=2e-3)
