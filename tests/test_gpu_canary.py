"""Out-of-bounds writes, caught without a sanitizer: every output and workspace
buffer the library is given sits between two 8 KB guard bands filled with a
known byte, and after each call the bands must be intact, the inputs
unchanged, and the results bit-identical to the same call on plain buffers.
Ragged lengths put the edges of every buffer next to a partial block.  (Runs
after the parity files.)"""
import numpy as np
import pytest
import torch

from test_gpu_parity import _custom, _inputs, _to_dev

pytestmark = pytest.mark.gpu

PAD = 8192          # guard bytes on each side; a multiple of 256 keeps the workspace alignment
CANARY = 0xA5
DEV = "cuda"


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


class Guarded:
    """A tensor of the given shape and dtype inside guard bands."""

    def __init__(self, shape, dtype):
        self.nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.buf = torch.full((self.nbytes + 2 * PAD,), CANARY, dtype=torch.uint8, device=DEV)
        self.t = self.buf[PAD:PAD + self.nbytes].view(dtype).view(*shape)

    def intact(self) -> bool:
        return bool((self.buf[:PAD] == CANARY).all()) and bool((self.buf[PAD + self.nbytes:] == CANARY).all())


def _ws(nbytes):
    return Guarded((max(int(nbytes), 256),), torch.uint8)


def _snapshot(d):
    return {k: v.clone() for k, v in d.items() if torch.is_tensor(v)}


def _unchanged(before, d):
    return all(torch.equal(before[k], d[k]) for k in before)


@pytest.mark.parametrize("theta,q_chunk", [(-1, 0), (0, 0), (-1, 700)])
def test_prefill_writes_stay_inside(M, theta, q_chunk):
    w = _custom("canary", 64, 4, 128, 64, 16, hot=0.05, seed=81)
    inp = _inputs(w, lengths=[1000, 257, 130, 2900], T_lens=[1000, 100, 130, 1777])
    shape, seqs, d = _to_dev(M, w, inp)
    before = _snapshot(d)
    T = seqs.total_q
    prev = M.msa_set_tile_threshold(theta)
    try:
        ref_sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
        ref_out, ref_lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], ref_sel, q_chunk=q_chunk)
        sel = Guarded((T, w.G, w.k), torch.int32)
        ws_i = _ws(M.msa_index_topk_workspace_size(shape, seqs))
        M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"], sel=sel.t, ws=ws_i.t)
        out = Guarded((T, w.H, w.d), torch.bfloat16)
        lse = Guarded((T, w.H), torch.float32)
        ws_a = _ws(M.msa_sparse_attn_workspace_size(shape, seqs, q_chunk))
        M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel.t, out=out.t, lse=lse.t,
                                  q_chunk=q_chunk, ws=ws_a.t)
    finally:
        M.msa_set_tile_threshold(prev)
    torch.cuda.synchronize()
    for name, g in (("sel", sel), ("index ws", ws_i), ("out", out), ("lse", lse), ("attention ws", ws_a)):
        assert g.intact(), f"{name}: guard band overwritten"
    assert _unchanged(before, d), "an input was modified"
    assert torch.equal(sel.t, ref_sel) and torch.equal(out.t, ref_out) and torch.equal(lse.t, ref_lse)


def test_decode_and_dense_writes_stay_inside(M):
    w = _custom("canary_dec", 64, 4, 128, 64, 16, hot=0.02, seed=82, kind="decode")
    inp = _inputs(w, lengths=[1, 127, 129, 4097, 9000])
    shape, seqs, d = _to_dev(M, w, inp)
    before = _snapshot(d)
    B = seqs.total_q
    ref_sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    ref_out, ref_lse = M.msa_sparse_attn_decode(shape, seqs, d["q"], d["k"], d["v"], ref_sel)
    sel = Guarded((B, w.G, w.k), torch.int32)
    ws_i = _ws(M.msa_index_topk_workspace_size(shape, seqs))
    M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"], sel=sel.t, ws=ws_i.t)
    out = Guarded((B, w.H, w.d), torch.bfloat16)
    lse = Guarded((B, w.H), torch.float32)
    ws_a = _ws(M.msa_sparse_attn_workspace_size(shape, seqs, 0))
    M.msa_sparse_attn_decode(shape, seqs, d["q"], d["k"], d["v"], sel.t, out=out.t, lse=lse.t, ws=ws_a.t)
    # dense causal attention of a ragged prefill
    wp = _custom("canary_dense", 64, 4, 128, 64, 16, seed=83)
    inp_p = _inputs(wp, lengths=[300, 1200, 77])
    shape_p, seqs_p, dp = _to_dev(M, wp, inp_p)
    ref_dense, ref_dlse = M.msa_dense_attn(shape_p, seqs_p, dp["q"], dp["k"], dp["v"], want_lse=True)
    T = seqs_p.total_q
    dout = Guarded((T, wp.H, wp.d), torch.bfloat16)
    dlse = Guarded((T, wp.H), torch.float32)
    ws_d = _ws(M.msa_dense_attn_workspace_size(shape_p, seqs_p))
    M.msa_dense_attn(shape_p, seqs_p, dp["q"], dp["k"], dp["v"], out=dout.t, lse=dlse.t, ws=ws_d.t)
    torch.cuda.synchronize()
    for name, g in (("sel", sel), ("index ws", ws_i), ("out", out), ("lse", lse), ("attention ws", ws_a),
                    ("dense out", dout), ("dense lse", dlse), ("dense ws", ws_d)):
        assert g.intact(), f"{name}: guard band overwritten"
    assert _unchanged(before, d), "an input was modified"
    assert torch.equal(sel.t, ref_sel) and torch.equal(out.t, ref_out) and torch.equal(lse.t, ref_lse)
    assert torch.equal(dout.t, ref_dense) and torch.equal(dlse.t, ref_dlse)


def test_paged_decode_and_combine_writes_stay_inside(M):
    from test_gpu_paged import _case
    w, inp, dev, shape, pages, (k_idx_p, k_p, v_p) = _case(M, [129, 5000, 127, 1, 300], seed=84)
    B = pages.batch
    ref_sel = M.msa_index_topk_decode_paged(shape, pages, dev["q_idx"], k_idx_p)
    ref_out, ref_lse = M.msa_sparse_attn_decode_paged(shape, pages, dev["q"], k_p, v_p, ref_sel)
    cache = {"k_idx": k_idx_p, "k": k_p, "v": v_p}
    before = _snapshot(cache)
    ws = _ws(M.msa_decode_paged_workspace_size(shape, pages))
    sel = Guarded((B, w.G, w.k), torch.int32)
    M.msa_index_topk_decode_paged(shape, pages, dev["q_idx"], k_idx_p, sel=sel.t, ws=ws.t)
    out = Guarded((B, w.H, w.d), torch.bfloat16)
    lse = Guarded((B, w.H), torch.float32)
    M.msa_sparse_attn_decode_paged(shape, pages, dev["q"], k_p, v_p, sel.t, out=out.t, lse=lse.t, ws=ws.t)
    # the stand-alone combine on hand-made partials
    H, G, dd, k, T = 8, 2, 64, 4, 37
    Hg = H // G
    gen = torch.Generator().manual_seed(85)
    acc = torch.randn(T, G, k, dd // 8, Hg, 8, generator=gen).half().to(DEV)
    plse = (torch.randn(T, G, k, Hg, generator=gen) * 3).float().to(DEV)
    csel = torch.randint(0, 50, (T, G, k), generator=gen, dtype=torch.int32).to(DEV)
    cshape = M.make_shape(H, G, dd, 32, k)
    ref_c, _ = M.msa_combine(cshape, T, acc, plse, csel)
    cout = Guarded((T, H, dd), torch.bfloat16)
    clse = Guarded((T, H), torch.float32)
    M.msa_combine(cshape, T, acc, plse, csel, out=cout.t, lse=clse.t)
    torch.cuda.synchronize()
    for name, g in (("sel", sel), ("ws", ws), ("out", out), ("lse", lse), ("combine out", cout),
                    ("combine lse", clse)):
        assert g.intact(), f"{name}: guard band overwritten"
    assert _unchanged(before, cache), "the paged cache was modified"
    assert torch.equal(sel.t, ref_sel) and torch.equal(out.t, ref_out) and torch.equal(lse.t, ref_lse)
    assert torch.equal(cout.t, ref_c)
