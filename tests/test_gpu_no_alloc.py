"""The allocation-free decode index entry point (fixed scratch array inside the
library, for callers that cannot allocate device memory at call time) gives
the same selection as the workspace entry point, on two calls in a row.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_long_exp_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _case(seed, lengths):
    w = W.Workload("noalloc", "decode", H=64, G=4, d=128, d_idx=64, B_k=128, k=16, seed=seed, hot_frac=0.02)
    inp = W.make_inputs(w, "cuda", lengths=lengths)
    return w, inp


def test_noalloc_decode_index_matches_workspace_entry_point():
    assert torch.cuda.is_available(), "GPU test"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    lib = msa.load_library()
    assert msa.msa_index_topk_decode_noalloc_max_scratch() == 16 << 20
    for seed, lengths in ((41, [129, 5000, 131072 + 5, 77, 1]), (42, [300000, 4096, 2049])):
        w, inp = _case(seed, lengths)
        shape = msa.make_shape(w.H, w.G, w.d, w.d_idx, w.k)
        seqs = msa.make_varlen(inp["cu_q"], inp["cu_k"], inp["cu_q_host"], inp["cu_k_host"])
        ref = msa.msa_index_topk(shape, seqs, inp["q_idx"], inp["k_idx"])
        sel = torch.full_like(ref, -7)
        err = torch.full((1,), 99, dtype=torch.int32, device="cuda")
        msa.msa_index_topk_decode_noalloc(shape, seqs, inp["q_idx"], inp["k_idx"], sel, device_error=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        np.testing.assert_array_equal(sel.cpu().numpy(), ref.cpu().numpy())


def test_noalloc_rejects_sizes_beyond_the_array():
    from block_sparse_long_exp_b200 import msa
    lib = msa.load_library()
    shape = msa.make_shape(64, 4, 128, 64, 16)
    cu = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    big = 1 << 30                                   # 1G-token cache: scratch need > 16 MiB
    cuk = torch.tensor([0, big], dtype=torch.int32, device="cuda")
    seqs = msa.Varlen(1, 1, big, 0, 1, big, cu.data_ptr(), cuk.data_ptr())
    rc = lib.msa_index_topk_decode_noalloc(ctypes.byref(shape), ctypes.byref(seqs), 256, 256, 256, None, None)
    assert rc == 3                                  # MSA_ERR_WORKSPACE, nothing launched
