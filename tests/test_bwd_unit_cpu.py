"""The Main Branch backward kernel's arithmetic (msa_bwd_unit.cuh), built for
the host with g++ and replayed phase by phase as the kernel's CTA runs it, on a
ragged varlen case whose support walks several 64-token chunks, against the
fp64 oracle (oracle/main_backward.py): dq, dk and dv for the sparse support
and the dense one.  Inputs are bf16 values; the forward's output is the
oracle's rounded to bf16, as the kernel would receive it, so D carries that
rounding."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

from oracle import main_backward as B
from oracle import msa_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_long_exp_b200", "csrc")


def _bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).bfloat16().view(torch.int16).numpy() \
        .astype(np.uint16)


def _bf(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).bfloat16().double().numpy()


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("needs g++")
    out = str(tmp_path_factory.mktemp("bwd") / "bwd_unit_host")
    subprocess.run(["g++", "-O2", "-std=c++17", "-Wall", "-Werror", f"-I{CSRC}",
                    os.path.join(ROOT, "tests", "c", "bwd_unit_host.cc"), "-o", out], check=True)
    return out


def _replay(exe, tmp_path, dense, seed, H, G, d, k, S_lens, T_lens, tol):
    B_k = 128
    rng = np.random.default_rng(seed)
    cu_k = np.concatenate([[0], np.cumsum(S_lens)]).astype(np.int32)
    cu_q = np.concatenate([[0], np.cumsum(T_lens)]).astype(np.int32)
    T, S = int(cu_q[-1]), int(cu_k[-1])
    q, kk, v = _bf(rng.standard_normal((T, H, d))), _bf(rng.standard_normal((S, G, d))), \
        _bf(rng.standard_normal((S, G, d)))
    dout = _bf(rng.standard_normal((T, H, d)))
    q_idx = rng.integers(-4, 5, size=(T, G, 32)).astype(np.float64)
    k_idx = rng.integers(-4, 5, size=(S, 32)).astype(np.float64)
    sel = O.index_topk(q_idx, k_idx, cu_q.tolist(), cu_k.tolist(), k, B_k)
    sm = d ** -0.5
    use = np.tile(np.arange(8, dtype=np.int32)[None, None, :], (T, G, 1)) if dense else sel
    o, lse = O.msa_forward_rows(q, kk, v, use, cu_q, cu_k, list(range(T)), B_k, sm)
    case = tmp_path / "case.bin"
    with open(case, "wb") as f:
        f.write(np.array([T, S, H, G, d, k, B_k, len(S_lens), int(dense)], np.int32).tobytes())
        f.write(np.array([sm], np.float32).tobytes())
        for a in (cu_q, cu_k):
            f.write(a.astype(np.int32).tobytes())
        for a in (q, kk, v):
            f.write(_bits(a).tobytes())
        f.write(sel.astype(np.int32).tobytes())
        f.write(_bits(o).tobytes())
        f.write(lse.astype(np.float32).tobytes())
        f.write(_bits(dout).tobytes())
    res = tmp_path / "grads.bin"
    r = subprocess.run([exe, str(case), str(res)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "bad 0" in r.stdout
    flat = np.fromfile(res, dtype=np.float32)
    n_q, n_kv = T * H * d, S * G * d
    got = (flat[:n_q].reshape(T, H, d), flat[n_q:n_q + n_kv].reshape(S, G, d), flat[n_q + n_kv:].reshape(S, G, d))
    want = B.main_branch_backward(q, kk, v, sel, dout, cu_q, cu_k, B_k, sm, dense=dense)
    for name, a, b in zip(("dq", "dk", "dv"), got, want):
        np.testing.assert_allclose(a, b, rtol=0, atol=tol * np.abs(b).max(), err_msg=name)


@pytest.mark.parametrize("dense", [False, True])
def test_bwd_unit_matches_the_oracle(exe, tmp_path, dense):
    _replay(exe, tmp_path, dense, 41, 8, 2, 64, 4, [700, 129, 460], [300, 5, 460], 3e-3)


# The largest group the kernel takes (16 heads, each thread keeping 16 dq
# outputs) at d = 128, and one head group of 4 heads whose support is the
# query's own block alone (k = 1).  The bound is the GPU test's: D = <dout, o>
# reads o rounded to bf16, and where dP - D cancels that rounding reaches a few
# parts in 10^3 of the largest gradient.
@pytest.mark.parametrize("H,G,d,k,S_lens,T_lens", [
    (32, 2, 128, 8, [1100, 70], [180, 70]),
    (4, 1, 64, 1, [334, 500], [166, 257]),
])
def test_bwd_unit_other_shapes(exe, tmp_path, H, G, d, k, S_lens, T_lens):
    _replay(exe, tmp_path, False, 43, H, G, d, k, S_lens, T_lens, 5e-3)
