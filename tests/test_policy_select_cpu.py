"""The scored selection policies as the kernel computes them (msa_policy_unit.cuh:
block scores by the largest raw index score, forced sink blocks and local
window, the rest by (score desc, id asc)), built for the host with g++, against
the selection-policy oracle (oracle/selection_policies.py) on a ragged varlen
case with integer index values (exact scores, many ties) and hot blocks, for
several sink and window sizes; with no sink and a one-block window it is the
final rule of oracle.msa_oracle.index_topk.  Plus the entry point's host
checks."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

from oracle import msa_oracle as O
from oracle import selection_policies as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_long_exp_b200", "csrc")


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("needs g++")
    out = str(tmp_path_factory.mktemp("pol") / "policy_host")
    subprocess.run(["g++", "-O2", "-std=c++17", "-Wall", "-Werror", f"-I{CSRC}",
                    os.path.join(ROOT, "tests", "c", "policy_host.cc"), "-o", out], check=True)
    return out


def _replay(exe, tmp_path, seed, G, d_idx, k, S_lens, T_lens, n_sink, n_local):
    B_k = 128
    rng = np.random.default_rng(seed)
    cu_k = np.concatenate([[0], np.cumsum(S_lens)]).astype(np.int32)
    cu_q = np.concatenate([[0], np.cumsum(T_lens)]).astype(np.int32)
    T, S = int(cu_q[-1]), int(cu_k[-1])
    q_idx = rng.integers(-2, 3, size=(T, G, d_idx)).astype(np.float32)
    k_idx = rng.integers(-2, 3, size=(S, d_idx)).astype(np.float32)
    k_idx[300:428] *= 3                                      # a hot block of the first sequence
    bits = lambda a: torch.from_numpy(a).bfloat16().view(torch.int16).numpy().astype(np.uint16)  # noqa: E731
    case = tmp_path / "case.bin"
    with open(case, "wb") as f:
        f.write(np.array([T, S, G, d_idx, k, B_k, len(S_lens), n_sink, n_local], np.int32).tobytes())
        f.write(cu_q.tobytes())
        f.write(cu_k.tobytes())
        f.write(bits(q_idx).tobytes())
        f.write(bits(k_idx).tobytes())
    res = tmp_path / "sel.bin"
    subprocess.run([exe, str(case), str(res)], check=True, timeout=300)
    got = np.fromfile(res, dtype=np.int32).reshape(T, G, k)
    want = P.index_topk_policy(q_idx, k_idx, cu_q.tolist(), cu_k.tolist(), k, B_k, n_sink, n_local)
    np.testing.assert_array_equal(got, want)
    if (n_sink, n_local) == (0, 1):
        np.testing.assert_array_equal(got, O.index_topk(q_idx, k_idx, cu_q.tolist(), cu_k.tolist(), k, B_k))


@pytest.mark.parametrize("n_sink,n_local", [(0, 1), (1, 1), (2, 3), (1, 7), (0, 4)])
def test_policy_matches_the_oracle(exe, tmp_path, n_sink, n_local):
    _replay(exe, tmp_path, 17, 2, 32, 8, [2500, 129, 1400], [700, 129, 300], n_sink, n_local)


# d_idx = 128 (the widest index row the kernel takes) with k = 1, where only the
# forced block can be chosen, and k = 32 (the largest k it takes) over a
# sequence of 47 blocks, so that scores still decide.
@pytest.mark.parametrize("G,d_idx,k,n_sink,n_local", [(1, 128, 1, 0, 1), (2, 128, 32, 0, 1), (2, 64, 32, 4, 8)])
def test_policy_other_shapes(exe, tmp_path, G, d_idx, k, n_sink, n_local):
    _replay(exe, tmp_path, 19, G, d_idx, k, [6000, 300], [200, 300], n_sink, n_local)


def test_policy_entry_point_host_checks():
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    lib = msa.load_library()
    shape = msa.make_shape(64, 4, 128, 64, 16)
    cu = (ctypes.c_int32 * 2)(0, 0)
    seqs = msa.Varlen(1, 300, 300, 0, 300, 300, ctypes.addressof(cu), ctypes.addressof(cu))
    for n_sink, n_local in ((-1, 1), (0, 0), (8, 9)):
        assert lib.msa_index_topk_policy(ctypes.byref(shape), ctypes.byref(seqs), n_sink, n_local, 256, 256, 256,
                                         256, 1 << 20, None) == 1
    long = msa.Varlen(1, 2, (1 << 20) + 1, 0, 2, (1 << 20) + 1, ctypes.addressof(cu), ctypes.addressof(cu))
    assert lib.msa_index_topk_policy(ctypes.byref(shape), ctypes.byref(long), 1, 1, 256, 256, 256, 256, 1 << 20,
                                     None) == 2
    assert lib.msa_index_topk_policy(ctypes.byref(shape), ctypes.byref(seqs), 1, 1, 256, 256, 256, 256, 16,
                                     None) == 3
