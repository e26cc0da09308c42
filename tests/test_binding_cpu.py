"""Host-side argument checks of the Python binding: every tensor handed to a
C entry point is checked for dtype, shape (the layout the kernels read),
contiguity and device before anything reaches the GPU, and a varlen
description is checked for consistent offsets.  No GPU is needed: the checks
raise MsaError with CPU tensors before any device work."""
import pytest
import torch


@pytest.fixture(scope="module")
def M():
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


H, G, d, d_idx, k = 8, 2, 64, 32, 4


def _seqs(M, T, S):
    """A Varlen description built directly (make_varlen wants device offsets)."""
    return M.Varlen(1, T, S, 0, T, S, 0, 0)


def _bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_make_varlen_checks_offsets(M):
    cu = torch.zeros(3, dtype=torch.int32)
    with pytest.raises(M.MsaError, match="batch \\+ 1"):
        M.make_varlen(cu, cu, [0, 5, 9], [0, 9])
    with pytest.raises(M.MsaError, match="start at 0"):
        M.make_varlen(cu, cu, [1, 5, 9], [0, 5, 9])
    with pytest.raises(M.MsaError, match="decrease"):
        M.make_varlen(cu, cu, [0, 5, 4], [0, 5, 9])
    with pytest.raises(M.MsaError, match="queries but"):
        M.make_varlen(cu, cu, [0, 6, 9], [0, 5, 9])          # T_0 = 6 > S_0 = 5
    with pytest.raises(M.MsaError, match="int32"):
        M.make_varlen(cu, cu, [0, 1], [0, 2 ** 31])
    # consistent offsets: the tensors are checked next (dtype, then device)
    with pytest.raises(M.MsaError, match="cu_q: dtype"):
        M.make_varlen(cu.long(), cu, [0, 5, 9], [0, 5, 9])
    with pytest.raises(M.MsaError, match="cu_k: shape"):
        M.make_varlen(cu, cu[:2], [0, 5, 9], [0, 5, 9])
    with pytest.raises(M.MsaError, match="CUDA"):
        M.make_varlen(cu, cu, [0, 5, 9], [0, 5, 9])


def test_index_topk_checks_its_tensors(M):
    shape = M.make_shape(H, G, d, d_idx, k)
    s = _seqs(M, 10, 30)
    ok_q, ok_k = _bf(10, G, d_idx), _bf(30, d_idx)
    with pytest.raises(M.MsaError, match="q_idx: shape"):
        M.msa_index_topk(shape, s, _bf(10, G + 1, d_idx), ok_k)
    with pytest.raises(M.MsaError, match="k_idx: dtype"):
        M.msa_index_topk(shape, s, ok_q, ok_k.float())
    with pytest.raises(M.MsaError, match="contiguous"):
        M.msa_index_topk(shape, s, _bf(10, d_idx, G).transpose(1, 2), ok_k)
    with pytest.raises(M.MsaError, match="sel: dtype"):
        M.msa_index_topk(shape, s, ok_q, ok_k, sel=torch.zeros(10, G, k, dtype=torch.int64))
    with pytest.raises(M.MsaError, match="sel: shape"):
        M.msa_index_topk(shape, s, ok_q, ok_k, sel=torch.zeros(10, G, k + 1, dtype=torch.int32))
    with pytest.raises(M.MsaError, match="CUDA"):          # well-formed, but on the CPU
        M.msa_index_topk(shape, s, ok_q, ok_k)


def test_attention_calls_check_their_tensors(M):
    shape = M.make_shape(H, G, d, d_idx, k)
    s = _seqs(M, 10, 30)
    q, kv, sel = _bf(10, H, d), _bf(30, G, d), torch.zeros(10, G, k, dtype=torch.int32)
    for call in (M.msa_sparse_attn_prefill, M.msa_sparse_attn_decode):
        with pytest.raises(M.MsaError, match="q: shape"):
            call(shape, s, _bf(10, H, d + 1), kv, kv, sel)
        with pytest.raises(M.MsaError, match="shape"):        # keys of another length
            call(shape, s, q, _bf(29, G, d), kv, sel)
        with pytest.raises(M.MsaError, match="sel: dtype"):
            call(shape, s, q, kv, kv, sel.float())
        with pytest.raises(M.MsaError, match="out: dtype"):
            call(shape, s, q, kv, kv, sel, out=torch.zeros(10, H, d))
        with pytest.raises(M.MsaError, match="lse: shape"):
            call(shape, s, q, kv, kv, sel, lse=torch.zeros(10, H + 1))
        with pytest.raises(M.MsaError, match="ws: expected"):
            call(shape, s, q, kv, kv, sel, ws=torch.zeros(8, 8, dtype=torch.uint8).t())
        with pytest.raises(M.MsaError, match="CUDA"):
            call(shape, s, q, kv, kv, sel)
    with pytest.raises(M.MsaError, match="v: shape"):
        M.msa_dense_attn(shape, s, q, kv, _bf(30, G, d, 1))
    with pytest.raises(M.MsaError, match="CUDA"):
        M.msa_dense_attn(shape, s, q, kv, kv)


def test_combine_checks_the_blocked_partials(M):
    shape = M.make_shape(H, G, d, d_idx, k)
    T, Hg = 5, H // G
    acc = torch.zeros(T, G, k, d // 8, Hg, 8, dtype=torch.float16)
    plse = torch.zeros(T, G, k, Hg)
    sel = torch.zeros(T, G, k, dtype=torch.int32)
    with pytest.raises(M.MsaError, match="part_acc: .* elements"):
        M.msa_combine(shape, T, acc[:, :, :, :4], plse, sel)
    with pytest.raises(M.MsaError, match="part_acc: dtype"):
        M.msa_combine(shape, T, acc.bfloat16(), plse, sel)
    with pytest.raises(M.MsaError, match="part_lse: .* elements"):
        M.msa_combine(shape, T, acc, plse[:4], sel)
    with pytest.raises(M.MsaError, match="multiple of G"):
        M.msa_combine(M.make_shape(H, 3, d, d_idx, k), T, acc, plse, sel)
    with pytest.raises(M.MsaError, match="CUDA"):
        M.msa_combine(shape, T, acc, plse, sel)


def test_paged_calls_check_their_tensors(M):
    shape = M.make_shape(H, G, d, d_idx, k)
    table = torch.zeros(3, 4, dtype=torch.int32)
    lens = torch.ones(3, dtype=torch.int32)
    with pytest.raises(M.MsaError, match="block_table"):
        M.make_paged(lens, table[0], 128, 12)
    with pytest.raises(M.MsaError, match="seqlens: shape"):
        M.make_paged(lens[:2], table, 128, 12)
    with pytest.raises(M.MsaError, match="CUDA"):
        M.make_paged(lens, table, 128, 12)
    pages = M.Paged(3, 4, 128, 0, 12, 0, 0)                   # 12 pages of 128 rows
    rows = 12 * 128
    with pytest.raises(M.MsaError, match="k_idx_pages: shape"):
        M.msa_index_topk_decode_paged(shape, pages, _bf(3, G, d_idx), _bf(rows - 1, d_idx))
    with pytest.raises(M.MsaError, match="q: shape"):
        M.msa_sparse_attn_decode_paged(shape, pages, _bf(4, H, d), _bf(rows, G, d), _bf(rows, G, d),
                                       torch.zeros(3, G, k, dtype=torch.int32))
    with pytest.raises(M.MsaError, match="CUDA"):
        M.msa_sparse_attn_decode_paged(shape, pages, _bf(3, H, d), _bf(rows, G, d), _bf(rows, G, d),
                                       torch.zeros(3, G, k, dtype=torch.int32))


def test_index_kl_checks_its_tensors(M):
    shape = M.make_shape(H, G, d, d_idx, k)
    s = _seqs(M, 10, 30)
    q, kv = _bf(10, H, d), _bf(30, G, d)
    qi, ki = _bf(10, G, d_idx), _bf(30, d_idx)
    sel = torch.zeros(10, G, k, dtype=torch.int32)
    lse = torch.zeros(10, H)
    with pytest.raises(M.MsaError, match="sel: a tensor is required"):
        M.msa_index_kl(shape, s, q, kv, qi, ki, None, lse, 0.5)
    with pytest.raises(M.MsaError, match="lse: shape"):
        M.msa_index_kl(shape, s, q, kv, qi, ki, sel, torch.zeros(10, G), 0.5)
    with pytest.raises(M.MsaError, match="kl: dtype"):
        M.msa_index_kl(shape, s, q, kv, qi, ki, sel, lse, 0.5, kl=torch.zeros(10, G, dtype=torch.float64))
    with pytest.raises(M.MsaError, match="CUDA"):
        M.msa_index_kl(shape, s, q, kv, qi, ki, None, lse, 0.5, dense=True)


def test_backward_checks_its_tensors(M):
    shape = M.make_shape(H, G, d, d_idx, k)
    s = _seqs(M, 10, 30)
    q, kv, sel = _bf(10, H, d), _bf(30, G, d), torch.zeros(10, G, k, dtype=torch.int32)
    lse = torch.zeros(10, H)
    with pytest.raises(M.MsaError, match="dout: shape"):
        M.msa_sparse_attn_backward(shape, s, q, kv, kv, sel, q, lse, _bf(10, H, d + 1))
    with pytest.raises(M.MsaError, match="out: dtype"):
        M.msa_sparse_attn_backward(shape, s, q, kv, kv, sel, q.float(), lse, q)
    with pytest.raises(M.MsaError, match="sel: a tensor is required"):
        M.msa_sparse_attn_backward(shape, s, q, kv, kv, None, q, lse, q)
    with pytest.raises(M.MsaError, match="CUDA"):
        M.msa_sparse_attn_backward(shape, s, q, kv, kv, None, q, lse, q, dense=True)


def test_gather_pages_checks_its_tensors(M):
    s = _seqs(M, 10, 300)
    table = torch.zeros(1, 3, dtype=torch.int32)
    pages = torch.zeros(4 * 128, G, d, dtype=torch.bfloat16)
    with pytest.raises(M.MsaError, match="block_table"):
        M.msa_gather_pages(s, table[0], 4, pages)
    with pytest.raises(M.MsaError, match="2 rows for 1"):
        M.msa_gather_pages(s, torch.zeros(2, 3, dtype=torch.int32), 4, pages)
    with pytest.raises(M.MsaError, match="num_pages"):
        M.msa_gather_pages(s, table, 5, pages)
    with pytest.raises(M.MsaError, match="CUDA"):
        M.msa_gather_pages(s, table, 4, pages)


def test_a_missing_library_fails_loudly(tmp_path):
    # no fallback: without the built library every call stops with an error
    from block_sparse_long_exp_b200 import msa as M
    saved = M._lib
    M._lib = None
    try:
        with pytest.raises(M.MsaError, match="no CPU fallback"):
            M.load_library(str(tmp_path / "libmsa.so"))
    finally:
        M._lib = saved
