"""The allocation-free decode index entry point, msa_index_topk_decode_noalloc.

Some callers cannot allocate device memory when they call into the library:
a serving loop whose framework reserves all device memory up front and hands
out no scratch buffers, or a host that keeps cudaMalloc off its decode path
because cudaMalloc synchronizes the whole device.  For them this entry point
keeps its scratch (block scores, offsets, error word) in a fixed array inside
the library.  Here it is called through the C ABI and must give the same
selection as the workspace entry point (msa_index_topk) and as the fp64 oracle
on several calls in a row, the array keeping the previous call's contents
between them.  Selections are integer block ids: the comparison is exact.

pytest collects this file last (tests/conftest.py puts it at the end of the
GPU run order), so a run that stops at its first failure has already run every
other test by the time it gets here.  It passes alone in a fresh process too.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import msa_oracle as O
from block_sparse_long_exp_b200 import workloads as W

pytestmark = pytest.mark.gpu

MSA_OK, MSA_ERR_WORKSPACE = 0, 3


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU test"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


def _case(seed, lengths):
    w = W.Workload("noalloc", "decode", H=64, G=4, d=128, d_idx=64, B_k=128, k=16, seed=seed, hot_frac=0.02)
    return w, W.make_inputs(w, "cuda", lengths=lengths)


def _oracle_sel(w, inp):
    return O.index_topk(inp["q_idx"].float().cpu().numpy(), inp["k_idx"].float().cpu().numpy(),
                        inp["cu_q_host"], inp["cu_k_host"], w.k, w.B_k)


def test_noalloc_matches_workspace_entry_point_and_oracle(M):
    assert M.msa_index_topk_decode_noalloc_max_scratch() == 16 << 20
    cases = [(41, [129, 5000, 131072 + 5, 77, 1]), (42, [300000, 4096, 2049]),
             (41, [129, 5000, 131072 + 5, 77, 1])]       # the first again, after a larger call
    for seed, lengths in cases:
        w, inp = _case(seed, lengths)
        shape = M.make_shape(w.H, w.G, w.d, w.d_idx, w.k)
        seqs = M.make_varlen(inp["cu_q"], inp["cu_k"], inp["cu_q_host"], inp["cu_k_host"])
        ref = M.msa_index_topk(shape, seqs, inp["q_idx"], inp["k_idx"])
        sel = torch.full_like(ref, -7)
        err = torch.full((1,), 99, dtype=torch.int32, device="cuda")
        M.msa_index_topk_decode_noalloc(shape, seqs, inp["q_idx"], inp["k_idx"], sel, device_error=err)
        torch.cuda.synchronize()
        assert int(err.item()) == MSA_OK
        got = sel.cpu().numpy()
        np.testing.assert_array_equal(got, ref.cpu().numpy())
        np.testing.assert_array_equal(got, _oracle_sel(w, inp))


def test_noalloc_no_queries_null_pointers(M):
    """A call with no queries succeeds without touching data (NULL pointers)."""
    lib = M.load_library()
    shape = M.make_shape(64, 4, 128, 64, 16)
    cu_q = torch.tensor([0, 0], dtype=torch.int32, device="cuda")
    cu_k = torch.tensor([0, 300], dtype=torch.int32, device="cuda")
    seqs = M.Varlen(1, 0, 300, 0, 0, 300, cu_q.data_ptr(), cu_k.data_ptr())
    err = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    rc = lib.msa_index_topk_decode_noalloc(ctypes.byref(shape), ctypes.byref(seqs), None, None, None,
                                           ctypes.c_void_p(err.data_ptr()), None)
    torch.cuda.synchronize()
    assert rc == MSA_OK and int(err.item()) == MSA_OK


def test_noalloc_rejects_sizes_beyond_the_array(M):
    """Just past the array (4*G bytes per cached block plus offsets): rejected
    before anything is launched; the dummy pointers are never dereferenced."""
    lib = M.load_library()
    shape = M.make_shape(64, 4, 128, 64, 16)
    cu = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    cap = M.msa_index_topk_decode_noalloc_max_scratch()
    for total_k in (134_217_856, 1 << 30):       # the first: 1,048,577 blocks, one more than fits
        cuk = torch.tensor([0, total_k], dtype=torch.int32, device="cuda")
        seqs = M.Varlen(1, 1, total_k, 0, 1, total_k, cu.data_ptr(), cuk.data_ptr())
        assert lib.msa_index_topk_workspace_size(ctypes.byref(shape), ctypes.byref(seqs)) > cap
        rc = lib.msa_index_topk_decode_noalloc(ctypes.byref(shape), ctypes.byref(seqs), 256, 256, 256, None, None)
        assert rc == MSA_ERR_WORKSPACE
