"""Decode over a paged KV cache (a page = one B_k-token block, pages in any
order, with unused pages of junk between them): the paged calls must give
exactly the packed calls' selection and output on the same tokens, and the
oracle's.  A page id outside the cache is reported, not read."""
import numpy as np
import pytest
import torch

from conftest import MAX_ABS_TOL, MEAN_REL_TOL, max_abs, mean_rel
from oracle import msa_oracle as O
from block_sparse_long_exp_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


def _to_pages(inp, w, spare, seed):
    """Copies the packed caches into pages in a random order."""
    cu_k = inp["cu_k_host"]
    batch = len(cu_k) - 1
    lens = [cu_k[b + 1] - cu_k[b] for b in range(batch)]
    nblk = [(L + w.B_k - 1) // w.B_k for L in lens]
    used = sum(nblk)
    num_pages = used + spare
    gen = torch.Generator().manual_seed(seed)
    perm = torch.randperm(num_pages, generator=gen)[:used].tolist()
    rows = num_pages * w.B_k
    k_idx_p = (torch.randn(rows, w.d_idx, generator=gen) * 50).bfloat16()      # junk outside the tokens
    k_p = (torch.randn(rows, w.G, w.d, generator=gen) * 50).bfloat16()
    v_p = (torch.randn(rows, w.G, w.d, generator=gen) * 50).bfloat16()
    table = torch.full((batch, max(nblk) + 1), -1, dtype=torch.int32)
    i = 0
    for b in range(batch):
        for j in range(nblk[b]):
            pg = perm[i]
            i += 1
            table[b, j] = pg
            r0 = cu_k[b] + j * w.B_k
            n = min(cu_k[b + 1], r0 + w.B_k) - r0
            dst = slice(pg * w.B_k, pg * w.B_k + n)
            k_idx_p[dst] = inp["k_idx"][r0:r0 + n]
            k_p[dst] = inp["k"][r0:r0 + n]
            v_p[dst] = inp["v"][r0:r0 + n]
    return k_idx_p, k_p, v_p, table, torch.tensor(lens, dtype=torch.int32), num_pages, max(lens)


def _case(M, lengths, seed):
    w = W.Workload("paged", "decode", H=64, G=4, d=128, d_idx=64, B_k=128, k=16, seed=seed, hot_frac=0.02)
    inp = W.make_inputs(w, "cpu", lengths=lengths)
    k_idx_p, k_p, v_p, table, lens, num_pages, max_len = _to_pages(inp, w, spare=7, seed=seed + 1)
    dev = {k: v.cuda() for k, v in inp.items() if torch.is_tensor(v)}
    shape = M.make_shape(w.H, w.G, w.d, w.d_idx, w.k)
    pages = M.make_paged(lens.cuda(), table.cuda(), max_len, num_pages)
    return w, inp, dev, shape, pages, (k_idx_p.cuda(), k_p.cuda(), v_p.cuda())


def test_paged_decode_equals_packed_and_oracle(M):
    lengths = [129, 5000, 127, 2048, 7777, 128, 1, 256 + 5]
    w, inp, dev, shape, pages, (k_idx_p, k_p, v_p) = _case(M, lengths, seed=61)
    # packed reference path
    seqs = M.make_varlen(dev["cu_q"], dev["cu_k"], inp["cu_q_host"], inp["cu_k_host"])
    sel_packed = M.msa_index_topk(shape, seqs, dev["q_idx"], dev["k_idx"])
    out_packed, lse_packed = M.msa_sparse_attn_decode(shape, seqs, dev["q"], dev["k"], dev["v"], sel_packed)
    # paged
    sel = M.msa_index_topk_decode_paged(shape, pages, dev["q_idx"], k_idx_p)
    out, lse = M.msa_sparse_attn_decode_paged(shape, pages, dev["q"], k_p, v_p, sel)
    torch.cuda.synchronize()
    assert torch.equal(sel, sel_packed)
    assert torch.equal(out, out_packed) and torch.equal(lse, lse_packed)
    # oracle
    f = lambda t: t.float().cpu().numpy()
    ref_sel = O.index_topk(f(inp["q_idx"]), f(inp["k_idx"]), inp["cu_q_host"], inp["cu_k_host"], w.k, w.B_k)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref_sel)
    T = inp["cu_q_host"][-1]
    o_ref, l_ref = O.msa_forward_rows(f(inp["q"]), f(inp["k"]), f(inp["v"]), ref_sel, inp["cu_q_host"],
                                      inp["cu_k_host"], list(range(T)), w.B_k, w.sm_scale)
    o = f(out)
    assert max_abs(o, o_ref) <= MAX_ABS_TOL and mean_rel(o, o_ref) <= MEAN_REL_TOL
    assert max_abs(f(lse), l_ref) <= 1e-3


def test_paged_bad_page_is_reported_not_read(M):
    lengths = [700, 300]
    w, inp, dev, shape, pages, (k_idx_p, k_p, v_p) = _case(M, lengths, seed=62)
    table = pages._keep[1].cpu().clone()
    table[0, 2] = pages.num_pages + 5                       # outside the cache
    bad = M.make_paged(pages._keep[0], table.cuda(), pages.max_seqlen, pages.num_pages)
    with pytest.raises(M.MsaError, match="DEVICE_CHECK"):
        M.msa_index_topk_decode_paged(shape, bad, dev["q_idx"], k_idx_p)
    # a selection of sequence 0 that names the bad block
    sel = M.msa_index_topk_decode_paged(shape, pages, dev["q_idx"], k_idx_p)
    sel[0, :, 0] = 2
    sel[0, :, 1:] = -1
    with pytest.raises(M.MsaError, match="DEVICE_CHECK"):
        M.msa_sparse_attn_decode_paged(shape, bad, dev["q"], k_p, v_p, sel)
    torch.cuda.synchronize()                                # the context is still usable
    M.msa_sparse_attn_decode_paged(shape, pages, dev["q"], k_p, v_p,
                                   M.msa_index_topk_decode_paged(shape, pages, dev["q_idx"], k_idx_p))
