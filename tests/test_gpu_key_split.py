"""Decode split by key range through the library on one GPU
(block_sparse_long_exp_b200/shard.py: each "rank" is run in turn on its key
slice).  Per slice msa_index_topk_decode_candidates gives the range's k-1
best blocks; msa_merge_candidates merges every slice's candidates into a
selection that must equal msa_index_topk's on the whole caches (and the
oracle's) bit for bit; per slice msa_select_block_range and
msa_sparse_attn_decode attend its own blocks; msa_combine merges the slices'
outputs (one slot per slice) within the main branch's tolerance of the
oracle."""
import numpy as np
import pytest
import torch

from block_sparse_long_exp_b200 import shard as SH
from block_sparse_long_exp_b200 import workloads as W
from test_gpu_parity import _check_out, _oracle_out, _oracle_sel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


@pytest.mark.parametrize("world,B_k", [(2, 128), (4, 128), (3, 64)])
def test_key_slices_give_the_whole_cache_result(M, world, B_k):
    w = W.Workload("keysplit_gpu", "decode", H=64, G=4, d=128, d_idx=64, B_k=B_k, k=16, seed=57, hot_frac=0.02)
    lengths = [200003, 9000, 40961, 1537]
    inp = W.make_inputs(w, "cuda", lengths=lengths)
    shape = M.make_shape(w.H, w.G, w.d, w.d_idx, w.k, B_k=B_k)
    seqs = M.make_varlen(inp["cu_q"], inp["cu_k"], inp["cu_q_host"], inp["cu_k_host"])
    whole = M.msa_index_topk(shape, seqs, inp["q_idx"], inp["k_idx"])
    cands_i, cands_s, parts = [], [], []
    for r in range(world):
        part = SH.key_slice(inp, lengths, r, world, B_k)
        seqs_r = M.make_varlen(part["cu_q"], part["cu_k"], part["cu_q_host"], part["cu_k_host"])
        ids, scores = M.msa_index_topk_decode_candidates(shape, seqs_r, inp["q_idx"], part["k_idx"],
                                                         part["all_blocks"])
        gi, gs = SH.gather_candidates(ids, scores, part["blk_lo"])
        cands_i.append(gi)
        cands_s.append(gs)
        parts.append((part, seqs_r))
    sel = M.msa_merge_candidates(shape, torch.cat(cands_i, dim=2).contiguous(), torch.cat(cands_s, dim=2).contiguous(),
                                 parts[-1][0]["local_block"])
    torch.cuda.synchronize()
    assert torch.equal(sel, whole)
    host = {kk: (v.cpu() if torch.is_tensor(v) else v) for kk, v in inp.items()}
    np.testing.assert_array_equal(sel.cpu().numpy(), _oracle_sel(w, host))
    outs, lses, sels = [], [], []
    for part, seqs_r in parts:
        sel_r = M.msa_select_block_range(shape, sel, part["blk_lo"], part["blk_hi"])
        out_r, lse_r = M.msa_sparse_attn_decode(shape, seqs_r, inp["q"], part["k"], part["v"], sel_r)
        outs.append(out_r)
        lses.append(lse_r)
        sels.append(sel_r)
    acc, plse, slot = SH.rank_partials(outs, lses, sels, w.H, w.G)
    cshape = M.make_shape(w.H, w.G, w.d, w.d_idx, world, B_k=B_k)
    lse = torch.empty((len(lengths), w.H), dtype=torch.float32, device="cuda")
    out, _ = M.msa_combine(cshape, len(lengths), acc, plse, slot, lse=lse)
    o_ref, l_ref = _oracle_out(w, host, sel.cpu().numpy())
    _check_out(out, lse, o_ref, l_ref)
