"""Group-sharded prefill through the library on one GPU: every rank's slice
(block_sparse_long_exp_b200/shard.py: G/N consecutive GQA groups with their
query heads, the index keys whole) run as a layer of G/N groups.  Each slice's
selection equals its groups' columns of the whole layer's, bit for bit, and
the outputs joined over the heads are within the main branch's tolerance of
the oracle.  (Runs after every other GPU test file.)"""
import numpy as np
import pytest
import torch

from block_sparse_long_exp_b200 import shard as SH
from test_gpu_parity import _check_out, _custom, _inputs, _oracle_out, _to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


@pytest.mark.parametrize("world", [2, 4])
def test_group_slices_equal_the_whole_layer(M, world):
    w = _custom("group_shard", 64, 4, 128, 64, 16, hot=0.05, seed=97)
    inp = _inputs(w, lengths=[2400, 300], T_lens=[700, 300])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    outs, lses = [], []
    for g0, g1 in SH.split_groups(w.G, world):
        part = SH.group_slice(d, w.H, w.G, g0, g1)
        shape_r = M.make_shape(w.H * (g1 - g0) // w.G, g1 - g0, w.d, w.d_idx, w.k)
        sel_r = M.msa_index_topk(shape_r, seqs, part["q_idx"], part["k_idx"])
        out_r, lse_r = M.msa_sparse_attn_prefill(shape_r, seqs, part["q"], part["k"], part["v"], sel_r)
        torch.cuda.synchronize()
        assert torch.equal(sel_r, sel[:, g0:g1])
        outs.append(out_r)
        lses.append(lse_r)
    out, lse = torch.cat(outs, dim=1), torch.cat(lses, dim=1)
    o_ref, l_ref = _oracle_out(w, inp, sel.cpu().numpy())
    _check_out(out, lse, o_ref, l_ref)
    assert out.shape == (inp["cu_q_host"][-1], w.H, w.d) and np.all(np.isfinite(lse.cpu().numpy()))
