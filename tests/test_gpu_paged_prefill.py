"""Prefill (and chunked prefill) over a paged KV cache on the GPU: the pages
(one B_k-token block each, in a random order, with junk pages between them)
gathered into packed rows by msa_gather_pages, then the packed calls; the
selection, output and log-sum-exp must equal the packed prefill's on the same
tokens bit for bit.  A page outside the cache is reported.  (Runs after the
parity files.)"""
import pytest
import torch

from test_gpu_paged import _to_pages
from test_gpu_parity import _custom, _inputs, _to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


def _case(M, seed, T_lens):
    w = _custom("paged_prefill", 64, 4, 128, 64, 16, hot=0.05, seed=seed)
    inp = _inputs(w, lengths=[1000, 257, 3000, 130], T_lens=T_lens)
    shape, seqs, d = _to_dev(M, w, inp)
    k_idx_p, k_p, v_p, table, _, num_pages, _ = _to_pages(inp, w, spare=9, seed=seed + 1)
    return w, shape, seqs, d, (k_idx_p.cuda(), k_p.cuda(), v_p.cuda(), table.cuda(), num_pages)


@pytest.mark.parametrize("T_lens", [[1000, 257, 3000, 130], [1000, 100, 1700, 130]])
def test_paged_prefill_equals_packed(M, T_lens):
    w, shape, seqs, d, (k_idx_p, k_p, v_p, table, num_pages) = _case(M, 95, T_lens)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
    assert torch.equal(M.msa_gather_pages(seqs, table, num_pages, k_p), d["k"])
    psel, pout, plse = M.msa_prefill_paged(shape, seqs, table, num_pages, d["q"], d["q_idx"], k_idx_p, k_p, v_p)
    torch.cuda.synchronize()
    assert torch.equal(psel, sel)
    assert torch.equal(pout, out) and torch.equal(plse, lse)


def test_gather_bad_page_is_reported(M):
    w, shape, seqs, d, (k_idx_p, k_p, v_p, table, num_pages) = _case(M, 96, [1000, 257, 3000, 130])
    bad = table.clone()
    bad[2, 5] = num_pages + 3                      # sequence 2 holds 24 blocks: block 5 is in use
    with pytest.raises(M.MsaError, match="DEVICE_CHECK"):
        M.msa_gather_pages(seqs, bad, num_pages, k_p)
    torch.cuda.synchronize()                       # the context is still usable
    M.msa_gather_pages(seqs, table, num_pages, k_p)
