"""The largest batches the calls take, against the oracle: a prefill of 1024
sequences (the prefill index kernel's limit) of 1-600 tokens each, so that
128-query tiles end at a sequence boundary almost everywhere, and a decode
of 2048 sequences (decode-shaped calls have no batch limit).  The prefill is
compared on sampled rows (each sequence's last row among them), the decode
on every row.  (Runs after the parity files.)"""
import numpy as np
import pytest
import torch

from conftest import MAX_ABS_TOL, MEAN_REL_TOL, max_abs, mean_rel
from oracle import msa_oracle as O
from test_gpu_parity import _custom, _f32, _inputs, _oracle_out, _oracle_sel, _to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


def _rows_oracle_sel(w, inp, rows):
    """Oracle selection of the listed rows only (prefill: position = row - cu_q[b])."""
    cu_q, cu_k = inp["cu_q_host"], inp["cu_k_host"]
    q_idx, k_idx = _f32(inp["q_idx"]), _f32(inp["k_idx"])
    out = np.full((len(rows), w.G, w.k), -1, dtype=np.int32)
    for i, t in enumerate(rows):
        b = int(np.searchsorted(cu_q, t, side="right") - 1)
        T_b, S_b = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        pos = S_b - T_b + (t - cu_q[b])
        out[i] = O.index_topk_rows(q_idx[t:t + 1], k_idx[cu_k[b]:cu_k[b + 1]], [pos], w.k, w.B_k)[0]
    return out


@pytest.mark.parametrize("theta", [-1, 0])
def test_prefill_1024_sequences(M, theta):
    w = _custom("maxbatch", 8, 2, 64, 32, 4, hot=0.02, seed=91)
    lengths = np.random.default_rng(91).integers(1, 601, size=1024).tolist()
    inp = _inputs(w, lengths=lengths)
    shape, seqs, d = _to_dev(M, w, inp)
    prev = M.msa_set_tile_threshold(theta)
    try:
        sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
        out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
    finally:
        M.msa_set_tile_threshold(prev)
    torch.cuda.synchronize()
    T = inp["cu_q_host"][-1]
    rng = np.random.default_rng(92)
    rows = sorted(set(rng.choice(T, 1500, replace=False).tolist())
                  | {inp["cu_q_host"][b + 1] - 1 for b in range(0, 1024, 5)})
    sel_np = sel.cpu().numpy()
    np.testing.assert_array_equal(sel_np[rows], _rows_oracle_sel(w, inp, rows))
    o_ref, l_ref = _oracle_out(w, inp, sel_np, rows)
    o = _f32(out)[rows]
    assert np.all(np.isfinite(o))
    assert max_abs(o, o_ref) <= MAX_ABS_TOL and mean_rel(o, o_ref) <= MEAN_REL_TOL
    assert max_abs(_f32(lse)[rows], l_ref) <= 1e-3


def test_decode_2048_sequences(M):
    w = _custom("maxbatch_dec", 8, 2, 64, 32, 4, hot=0.02, seed=93, kind="decode")
    lengths = np.random.default_rng(93).integers(1, 1201, size=2048).tolist()
    inp = _inputs(w, lengths=lengths)
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_index_topk(shape, seqs, d["q_idx"], d["k_idx"])
    out, lse = M.msa_sparse_attn_decode(shape, seqs, d["q"], d["k"], d["v"], sel)
    torch.cuda.synchronize()
    ref = _oracle_sel(w, inp)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref)
    o_ref, l_ref = _oracle_out(w, inp, ref)
    o = _f32(out)
    assert np.all(np.isfinite(o))
    assert max_abs(o, o_ref) <= MAX_ABS_TOL and mean_rel(o, o_ref) <= MEAN_REL_TOL
    assert max_abs(_f32(lse), l_ref) <= 1e-3
