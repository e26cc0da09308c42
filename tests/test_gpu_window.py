"""The FLOP-matched sliding-window baseline on the GPU: msa_select_window's
selection equals the selection-policy oracle's fixed pattern on every row
(prefill with the queries as the last T_b tokens, and decode), and the
main-branch calls run it: their output matches the fp64 oracle on that
selection.  (Runs after the parity files.)"""
import numpy as np
import pytest
import torch

from oracle import msa_oracle as O
from oracle import selection_policies as P
from test_gpu_parity import _check_out, _custom, _inputs, _oracle_out, _to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


def _oracle_window(w, inp, n_sink):
    cu_q, cu_k = inp["cu_q_host"], inp["cu_k_host"]
    T = cu_q[-1]
    out = np.full((T, w.G, w.k), -1, dtype=np.int32)
    for b in range(len(cu_q) - 1):
        for i, pos in enumerate(O.query_positions(cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b])):
            lb = int(pos) // w.B_k
            blocks = P.select_blocks_policy(np.zeros(lb + 1), w.k, n_sink, w.k - n_sink)
            out[cu_q[b] + i, :, :len(blocks)] = blocks
    return out


@pytest.mark.parametrize("n_sink", [1, 0, 3])
def test_window_prefill_selection_and_attention(M, n_sink):
    w = _custom("window", 64, 4, 128, 64, 16, seed=99)
    inp = _inputs(w, lengths=[3000, 129, 1900], T_lens=[900, 129, 700])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_select_window(shape, seqs, n_sink)
    ref = _oracle_window(w, inp, n_sink)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref)
    out, lse = M.msa_sparse_attn_prefill(shape, seqs, d["q"], d["k"], d["v"], sel)
    torch.cuda.synchronize()
    o_ref, l_ref = _oracle_out(w, inp, ref)
    _check_out(out, lse, o_ref, l_ref)


def test_window_decode_selection_and_attention(M):
    w = _custom("window_dec", 64, 4, 128, 64, 16, seed=98, kind="decode")
    inp = _inputs(w, lengths=[1, 128, 129, 2100, 5000])
    shape, seqs, d = _to_dev(M, w, inp)
    sel = M.msa_select_window(shape, seqs, 1)
    ref = _oracle_window(w, inp, 1)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref)
    out, lse = M.msa_sparse_attn_decode(shape, seqs, d["q"], d["k"], d["v"], sel)
    torch.cuda.synchronize()
    o_ref, l_ref = _oracle_out(w, inp, ref)
    _check_out(out, lse, o_ref, l_ref)
