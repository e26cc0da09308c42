"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle, at
sizes the oracle finishes in seconds: every row compared, several 128-query
tiles and ragged tails.  Selections must match exactly; outputs within
max-abs 2e-2 and mean-relative 5e-3 of fp64."""

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


def _f32(t):
    return t.float().cpu().numpy()


def _custom(name, H, G, d, d_idx, k, hot=0.0, seed=7, kind="prefill"):
    return W.Workload(name, kind, H=H, G=G, d=d, d_idx=d_idx, B_k=128, k=k, seed=seed, hot_frac=hot)


def _inputs(w, lengths=None, T_lens=None, T_override=None):
    """CPU draws; optional T_lens makes queries the last T_b tokens."""
    inp = W.make_inputs(w, "cpu", T_override=T_override, lengths=lengths)
    if T_lens is not None:
        # keep the last T_b query rows of each sequence
        cu_k = inp["cu_k_host"]
        rows = []
        cu_q = [0]
        for b, Tb in enumerate(T_lens):
            S_b = cu_k[b + 1] - cu_k[b]
            q0 = inp["cu_q_host"][b]
            rows.extend(range(q0 + S_b - Tb, q0 + S_b))
            cu_q.append(cu_q[-1] + Tb)
        idx = torch.tensor(rows, dtype=torch.long)
        inp["q"] = inp["q"][idx].contiguous()
        inp["q_idx"] = inp["q_idx"][idx].contiguous()
        inp["cu_q_host"] = cu_q
        inp["cu_q"] = torch.tensor(cu_q, dtype=torch.int32)
    return inp


def _to_dev(M, w, inp):
    d = {k: v.cuda() for k, v in inp.items() if torch.is_tensor(v)}
    shape = M.make_shape(w.H, w.G, w.d, w.d_idx, w.k, B_k=w.B_k)
    seqs = M.make_varlen(d["cu_q"], d["cu_k"], inp["cu_q_host"], inp["cu_k_host"])
    return shape, seqs, d


def _oracle_sel(w, inp):
    return O.index_topk(_f32(inp["q_idx"]), _f32(inp["k_idx"]), inp["cu_q_host"], inp["cu_k_host"], w.k, w.B_k)


def _check_out(o_gpu, lse_gpu, o_ref, lse_ref):
    o = _f32(o_gpu)
    assert np.all(np.isfinite(o))
    ma, mr = max_abs(o, o_ref), mean_rel(o, o_ref)
    assert ma <= MAX_ABS_TOL and mr <= MEAN_REL_TOL, (ma, mr)
    if lse_gpu is not None:
        assert max_abs(_f32(lse_gpu), lse_ref) <= 1e-3


# ------------------------------------------------------------ selection ----

def test_index_topk_tiny_exact(M):
    w = W.WORKLOADS["tiny_n4096"]
    inp = _inputs(w)
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    ref = _oracle_sel(w, inp)
    got = sel.cpu().numpy()
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} mismatches, first {bad[:5].tolist()}"


@pytest.mark.parametrize("hot", [0.0, 0.05])
def test_index_topk_varlen_ragged_exact(M, hot):
    w = _custom("ragged", 64, 4, 128, 64, 16, hot=hot, seed=11)
    inp = _inputs(w, lengths=[1000, 2817, 130, 64])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    np.testing.assert_array_equal(sel.cpu().numpy(), _oracle_sel(w, inp))


def test_index_topk_chunked_queries_exact(M):
    """Queries are the last T_b tokens of each sequence (chunk of a prefill)."""
    w = _custom("chunk", 64, 4, 128, 64, 16, seed=12)
    inp = _inputs(w, lengths=[3000, 1500, 2100], T_lens=[1200, 1500, 77])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    np.testing.assert_array_equal(sel.cpu().numpy(), _oracle_sel(w, inp))


def test_index_topk_decode_exact(M):
    """Decode-shaped call (one query per sequence): split scan + merge."""
    w = _custom("dec", 64, 4, 128, 64, 16, hot=0.02, seed=13, kind="decode")
    inp = _inputs(w, lengths=[129, 4096 + 77, 127, 2048, 9000, 1])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    np.testing.assert_array_equal(sel.cpu().numpy(), _oracle_sel(w, inp))


def test_index_topk_small_heads_and_k(M):
    """G = 1 and G = 2 variants, d_idx 128, k = 4."""
    for (H, G, d_idx, k) in [(16, 1, 128, 4), (8, 2, 64, 5)]:
        w = _custom("var", H, G, 64, d_idx, k, seed=14)
        inp = _inputs(w, lengths=[1500, 700])
        shape, seqs, d = _to_dev(M, w, inp)
        sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
        np.testing.assert_array_equal(sel.cpu().numpy(), _oracle_sel(w, inp))


# ------------------------------------------------------------ attention ----

def _oracle_out(w, inp, sel, rows=None):
    T = inp["cu_q_host"][-1]
    rows = list(range(T)) if rows is None else rows
    return O.msa_forward_rows(_f32(inp["q"]), _f32(inp["k"]), _f32(inp["v"]), sel, inp["cu_q_host"],
                              inp["cu_k_host"], rows, w.B_k, w.sm_scale)


def test_sparse_attn_tiny(M):
    w = W.WORKLOADS["tiny_n4096"]
    inp = _inputs(w)
    shape, seqs, d = _to_dev(M, w, inp)
    ref_sel = _oracle_sel(w, inp)
    sel = torch.from_numpy(ref_sel).cuda()
    out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
    o_ref, lse_ref = _oracle_out(w, inp, ref_sel)
    _check_out(out, lse, o_ref, lse_ref)


@pytest.mark.parametrize("q_chunk", [0, 700])
def test_sparse_attn_varlen_chunked(M, q_chunk):
    w = _custom("attn", 64, 4, 128, 64, 16, hot=0.05, seed=21)
    inp = _inputs(w, lengths=[2600, 130, 1901])
    shape, seqs, d = _to_dev(M, w, inp)
    ref_sel = _oracle_sel(w, inp)
    sel = torch.from_numpy(ref_sel).cuda()
    out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel, q_chunk=q_chunk)
    o_ref, lse_ref = _oracle_out(w, inp, ref_sel)
    _check_out(out, lse, o_ref, lse_ref)


def test_sparse_attn_queries_are_last_tokens(M):
    w = _custom("attn_chunk", 64, 4, 128, 64, 16, seed=22)
    inp = _inputs(w, lengths=[2000, 1300], T_lens=[300, 1300])
    shape, seqs, d = _to_dev(M, w, inp)
    ref_sel = _oracle_sel(w, inp)
    out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], torch.from_numpy(ref_sel).cuda())
    o_ref, lse_ref = _oracle_out(w, inp, ref_sel)
    _check_out(out, lse, o_ref, lse_ref)


def test_dense_special_case_on_gpu(M):
    """k >= number of causal blocks: every block is selected (dense causal GQA)."""
    w = _custom("dense_k", 16, 2, 64, 32, 32, seed=23)
    inp = _inputs(w, lengths=[3000])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    s = sel.cpu().numpy()
    for t in (0, 127, 128, 2999):
        nb = t // 128 + 1
        assert s[t, 0, :nb].tolist() == list(range(nb)) and np.all(s[t, 0, nb:] == -1)
    out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
    o_ref, lse_ref = _oracle_out(w, inp, s)
    _check_out(out, lse, o_ref, lse_ref)


def test_small_heads_attention(M):
    for (H, G, d_, k) in [(16, 1, 64, 4), (8, 2, 128, 6)]:
        w = _custom("small", H, G, d_, 32, k, seed=24)
        inp = _inputs(w, lengths=[1500, 333])
        shape, seqs, d = _to_dev(M, w, inp)
        ref_sel = _oracle_sel(w, inp)
        out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], torch.from_numpy(ref_sel).cuda())
        o_ref, lse_ref = _oracle_out(w, inp, ref_sel)
        _check_out(out, lse, o_ref, lse_ref)


def test_decode_end_to_end(M):
    w = _custom("dec2", 64, 4, 128, 64, 16, hot=0.02, seed=25, kind="decode")
    inp = _inputs(w, lengths=[129, 5000, 127, 2048, 7777])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    ref_sel = _oracle_sel(w, inp)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref_sel)
    out, lse = M.msa_sparse_attn_decode(shape, seqs, d["q"], d["k"], d["v"], sel)
    o_ref, lse_ref = _oracle_out(w, inp, ref_sel)
    _check_out(out, lse, o_ref, lse_ref)


def test_combine_entry_point(M):
    """msa_combine on hand-made partials against the oracle's log-sum-exp merge."""
    H, G, d_, k, T = 8, 2, 64, 4, 37
    Hg = H // G
    gen = torch.Generator().manual_seed(3)
    acc = torch.randn(T, G, k, Hg, d_, generator=gen).half()
    # device layout: [T, G, k, d/8, Hg, 8]
    acc_dev = acc.view(T, G, k, Hg, d_ // 8, 8).permute(0, 1, 2, 4, 3, 5).contiguous()
    plse = (torch.randn(T, G, k, Hg, generator=gen) * 3).float()
    sel = torch.randint(0, 50, (T, G, k), generator=gen, dtype=torch.int32)
    sel[::3, :, k - 1] = -1                      # some empty slots
    shape = M.make_shape(H, G, d_, 32, k)
    lse_out = torch.empty(T, H, device="cuda")
    out, _ = M.msa_combine(shape, T, acc_dev.cuda(), plse.cuda(), sel.cuda(), lse=lse_out)
    o = _f32(out)
    for t in range(T):
        for h in range(H):
            g, i = h // Hg, h % Hg
            slots = [s for s in range(k) if sel[t, g, s] >= 0]
            ro, rl = O.lse_combine(acc[t, g, slots, i].double().numpy(), plse[t, g, slots, i].double().numpy())
            assert np.max(np.abs(o[t, h] - ro)) <= 1e-2
            assert abs(lse_out[t, h].item() - rl) <= 1e-4


def test_combine_ignores_unused_slots(M):
    """Slots with sel < 0 take no part in the merge whatever their buffers
    hold: NaN partials and log-sum-exps there leave the result unchanged."""
    H, G, d_, k, T = 16, 2, 64, 5, 29
    Hg = H // G
    gen = torch.Generator().manual_seed(4)
    acc = torch.randn(T, G, k, Hg, d_, generator=gen).half()
    plse = (torch.randn(T, G, k, Hg, generator=gen) * 3).float()
    sel = torch.randint(0, 50, (T, G, k), generator=gen, dtype=torch.int32)
    sel[::2, :, 0] = -1
    sel[1::3, :, k - 1] = -1
    unused = (sel < 0)[:, :, :, None]
    acc = torch.where(unused[..., None], torch.full_like(acc, float("nan")), acc)
    plse = torch.where(unused, torch.full_like(plse, float("nan")), plse)
    acc_dev = acc.view(T, G, k, Hg, d_ // 8, 8).permute(0, 1, 2, 4, 3, 5).contiguous()
    shape = M.make_shape(H, G, d_, 32, k)
    lse_out = torch.empty(T, H, device="cuda")
    out, _ = M.msa_combine(shape, T, acc_dev.cuda(), plse.cuda(), sel.cuda(), lse=lse_out)
    o = _f32(out)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse_out.cpu().numpy()))
    for t in range(T):
        for h in range(H):
            g, i = h // Hg, h % Hg
            slots = [s_ for s_ in range(k) if sel[t, g, s_] >= 0]
            ro, rl = O.lse_combine(acc[t, g, slots, i].double().numpy(), plse[t, g, slots, i].double().numpy())
            assert np.max(np.abs(o[t, h] - ro)) <= 1e-2
            assert abs(lse_out[t, h].item() - rl) <= 1e-4


# ------------------------------------------- query tiles and dense GQA ----

def _prefill_with_threshold(M, theta, shape, seqs, d, sel, q_chunk=0):
    prev = M.msa_set_tile_threshold(theta)
    try:
        return M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel, q_chunk=q_chunk)
    finally:
        M.msa_set_tile_threshold(prev)


@pytest.mark.parametrize("theta", [0, 1, 3, -1, 1000])
def test_prefill_tile_threshold(M, theta):
    """Every split of the selections between query tiles and KV-outer lists
    gives the oracle's result: 0 (all KV-outer), 1 (every selected block of a
    tile), 3, automatic, and a threshold no block reaches.  Hot blocks, ragged
    tails, tiles that straddle a sequence boundary, queries that are the last
    tokens of their sequence."""
    w = _custom("tiles", 64, 4, 128, 64, 16, hot=0.05, seed=31)
    inp = _inputs(w, lengths=[2600, 130, 1901], T_lens=[2600, 130, 1001])
    shape, seqs, d = _to_dev(M, w, inp)
    ref_sel = _oracle_sel(w, inp)
    out, lse = _prefill_with_threshold(M, theta, shape, seqs, d, torch.from_numpy(ref_sel).cuda())
    o_ref, lse_ref = _oracle_out(w, inp, ref_sel)
    _check_out(out, lse, o_ref, lse_ref)


@pytest.mark.parametrize("theta", [1, -1])
def test_prefill_tiles_chunked_passes(M, theta):
    """Passes of 700 rows: tiles restart at each pass start."""
    w = _custom("tiles_q", 64, 4, 128, 64, 16, hot=0.05, seed=32)
    inp = _inputs(w, lengths=[3001, 1500])
    shape, seqs, d = _to_dev(M, w, inp)
    ref_sel = _oracle_sel(w, inp)
    out, lse = _prefill_with_threshold(M, theta, shape, seqs, d, torch.from_numpy(ref_sel).cuda(), q_chunk=700)
    o_ref, lse_ref = _oracle_out(w, inp, ref_sel)
    _check_out(out, lse, o_ref, lse_ref)


@pytest.mark.parametrize("theta", [1, -1])
def test_prefill_tiles_small_heads(M, theta):
    """H/G = 16, 4 and 8 (tiles of 16, 32, 32 queries), d = 64 and 128."""
    for (H, G, d_, k) in [(16, 1, 64, 4), (8, 2, 128, 6), (32, 4, 64, 8)]:
        w = _custom("tiles_small", H, G, d_, 32, k, hot=0.05, seed=33)
        inp = _inputs(w, lengths=[1500, 333])
        shape, seqs, d = _to_dev(M, w, inp)
        ref_sel = _oracle_sel(w, inp)
        out, lse = _prefill_with_threshold(M, theta, shape, seqs, d, torch.from_numpy(ref_sel).cuda())
        o_ref, lse_ref = _oracle_out(w, inp, ref_sel)
        _check_out(out, lse, o_ref, lse_ref)


def _all_blocks_sel(cu_q, cu_k, G, B_k=128):
    """Selection of every causal block (k >= blocks): the oracle's dense case."""
    T = cu_q[-1]
    nbmax = max((cu_k[b + 1] - cu_k[b] + B_k - 1) // B_k for b in range(len(cu_q) - 1))
    sel = np.full((T, G, nbmax), -1, dtype=np.int32)
    for b in range(len(cu_q) - 1):
        Tb, Sb = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        for i in range(Tb):
            nb = (Sb - Tb + i) // B_k + 1
            sel[cu_q[b] + i, :, :nb] = np.arange(nb)
    return sel


@pytest.mark.parametrize("H,G,d_", [(64, 4, 128), (16, 2, 64), (8, 2, 128), (32, 4, 64)])
def test_dense_causal_gqa(M, H, G, d_):
    """msa_dense_attn against the oracle with every causal block selected."""
    w = _custom("dense", H, G, d_, 32, 4, seed=41)
    inp = _inputs(w, lengths=[1500, 129, 700], T_lens=[1500, 129, 301])
    shape, seqs, d = _to_dev(M, w, inp)
    out, lse = M.msa_dense_attn(shape, seqs, d["q"], d["k"], d["v"], want_lse=True)
    sel = _all_blocks_sel(inp["cu_q_host"], inp["cu_k_host"], G)
    o_ref, lse_ref = _oracle_out(w, inp, sel)
    _check_out(out, lse, o_ref, lse_ref)


# ------------------------------------------------------------ errors -------

def test_out_of_range_selection_is_reported_not_faulted(M):
    w = _custom("bad", 64, 4, 128, 64, 16, seed=26)
    inp = _inputs(w, lengths=[600])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = torch.from_numpy(_oracle_sel(w, inp)).cuda()
    sel[10, 1, 0] = 3          # query 10 sits in block 0: block 3 is in its future
    with pytest.raises(M.MsaError, match="DEVICE_CHECK"):
        M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
    torch.cuda.synchronize()   # the context is still usable
    sel2 = torch.from_numpy(_oracle_sel(w, inp)).cuda()
    M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel2)


def test_workspace_too_small_is_rejected(M):
    w = _custom("ws", 64, 4, 128, 64, 16, seed=27)
    inp = _inputs(w, lengths=[300])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(M.MsaError, match="WORKSPACE"):
        M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel, ws=ws)
