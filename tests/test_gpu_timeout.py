"""Failure detection without a GPU fault: every spin-wait in the kernels gives
up after a bounded time and records MSA_ERR_TIMEOUT instead of hanging.  The
self-test kernel runs the library's own two kinds of wait (an mbarrier phase,
a counter other CTAs advance) on objects that nothing ever signals, with a
2 ms limit.  Both must run out, the status must read MSA_ERR_TIMEOUT at the
self-test's site, and the same context must then run a normal call correctly."""
import numpy as np
import pytest
import torch

from oracle import msa_oracle as O
from block_sparse_long_exp_b200 import workloads as W

pytestmark = pytest.mark.gpu

MSA_ERR_TIMEOUT = 5
SITE_SELFTEST = 221


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU test"
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    msa.load_library()
    return msa


def test_waits_run_out_and_the_context_stays_usable(M):
    for limit_us in (2000, 50):
        code, where, timed_out, _ = M.msa_selftest_wait_timeout(limit_us)
        assert code == MSA_ERR_TIMEOUT and where == SITE_SELFTEST and timed_out == 2
    # the context is still usable: a normal call gives the oracle's selection
    w = W.Workload("after_timeout", "prefill", H=8, G=2, d=64, d_idx=32, B_k=128, k=8, seed=3, T=1000)
    inp = W.make_inputs(w, "cuda")
    shape = M.make_shape(w.H, w.G, w.d, w.d_idx, w.k)
    seqs = M.make_varlen(inp["cu_q"], inp["cu_k"], inp["cu_q_host"], inp["cu_k_host"])
    sel = M.msa_index_topk(shape, seqs, inp["q_idx"], inp["k_idx"])
    ref = O.index_topk(inp["q_idx"].float().cpu().numpy(), inp["k_idx"].float().cpu().numpy(),
                       inp["cu_q_host"], inp["cu_k_host"], w.k, w.B_k)
    np.testing.assert_array_equal(sel.cpu().numpy(), ref)
