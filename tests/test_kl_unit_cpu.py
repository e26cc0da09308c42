"""The index-alignment kernels' arithmetic (msa_kl_unit.cuh: per-thread
partial sums over a CTA's share of the support, then their merge; the
gradient pass with the teacher held constant), built for
the host with g++ and run on a ragged varlen case for CTAs of 128 and of 7
threads, against the fp64 oracle of the same target (oracle/index_kl.py), for
the sparse support and the dense (warmup) one: the KL and its gradient with
respect to the index query and keys.  Inputs are bf16 values and the
log-sum-exps are the oracle's over the same support, so what differs is fp32
accumulation only."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

from oracle import index_kl as K
from oracle import msa_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_long_exp_b200", "csrc")


def _bf16_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).bfloat16().view(torch.int16).numpy() \
        .astype(np.uint16)


def _bf16_values(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).bfloat16().double().numpy()


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    if shutil.which("g++") is None:
        pytest.skip("needs g++")
    out = str(tmp_path_factory.mktemp("kl") / "kl_unit_host")
    subprocess.run(["g++", "-O2", "-std=c++17", "-Wall", "-Werror", f"-I{CSRC}",
                    os.path.join(ROOT, "tests", "c", "kl_unit_host.cc"), "-o", out], check=True)
    return out


def _replay(exe, tmp_path, dense, seed, H, G, d, d_idx, k, S_lens, T_lens):
    B_k = 128
    rng = np.random.default_rng(seed)
    cu_k = np.concatenate([[0], np.cumsum(S_lens)]).astype(np.int32)
    cu_q = np.concatenate([[0], np.cumsum(T_lens)]).astype(np.int32)
    T, S = int(cu_q[-1]), int(cu_k[-1])
    q = _bf16_values(rng.standard_normal((T, H, d)))
    kk = _bf16_values(rng.standard_normal((S, G, d)))
    q_idx = rng.integers(-4, 5, size=(T, G, d_idx)).astype(np.float64)
    k_idx = rng.integers(-4, 5, size=(S, d_idx)).astype(np.float64)
    sel = O.index_topk(q_idx, k_idx, cu_q.tolist(), cu_k.tolist(), k, B_k)
    sm, tau = d ** -0.5, 0.125
    rows = list(range(T))
    if dense:
        n_blk = (max(S_lens) + B_k - 1) // B_k
        every = np.tile(np.arange(n_blk, dtype=np.int32)[None, None, :], (T, G, 1))
        _, lse = O.msa_forward_rows(q, kk, np.zeros_like(kk), every, cu_q, cu_k, rows, B_k, sm)
    else:
        _, lse = O.msa_forward_rows(q, kk, np.zeros_like(kk), sel, cu_q, cu_k, rows, B_k, sm)
    case = tmp_path / "case.bin"
    with open(case, "wb") as f:
        f.write(np.array([T, S, H, G, d, d_idx, k, B_k, len(S_lens), int(dense)], np.int32).tobytes())
        f.write(np.array([sm, tau], np.float32).tobytes())
        for a in (cu_q, cu_k):
            f.write(a.astype(np.int32).tobytes())
        for a in (q, kk, q_idx, k_idx):
            f.write(_bf16_bits(a).tobytes())
        f.write(sel.astype(np.int32).tobytes())
        f.write(lse.astype(np.float32).tobytes())
    res = tmp_path / "kl.bin"
    r = subprocess.run([exe, str(case), str(res)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "bad 0" in r.stdout
    flat = np.fromfile(res, dtype=np.float32)
    n_kl, n_dq = 2 * T * G, 2 * T * G * d_idx
    got = flat[:n_kl].reshape(2, T, G)
    got_dq = flat[n_kl:n_kl + n_dq].reshape(2, T, G, d_idx)
    got_dk = flat[n_kl + n_dq:].reshape(2, S, d_idx)
    want = K.index_kl_rows(q, kk, q_idx, k_idx, sel, cu_q, cu_k, rows, B_k, sm, tau, dense=dense)
    assert np.all(want > -1e-9)
    _, want_dq, want_dk = K.index_kl_loss_and_grad(q, kk, q_idx, k_idx, sel, cu_q, cu_k, B_k, sm, tau, dense=dense)
    for cta in range(2):
        np.testing.assert_allclose(got[cta], want, rtol=2e-4, atol=2e-4)
        # gradients: fp32 sums of up to 2048 terms of magnitude ~tau * 4
        scale = np.abs(want_dq).max()
        np.testing.assert_allclose(got_dq[cta], want_dq, rtol=0, atol=2e-4 * scale)
        np.testing.assert_allclose(got_dk[cta], want_dk, rtol=0, atol=2e-4 * np.abs(want_dk).max())


@pytest.mark.parametrize("dense", [False, True])
def test_kl_unit_matches_the_oracle(exe, tmp_path, dense):
    _replay(exe, tmp_path, dense, 31, 8, 2, 64, 32, 4, [700, 129, 1000], [700, 5, 300])


# The largest group the kernels take (16 heads) with d = d_idx = 128, and a
# group of 4 heads whose support is the query's own block alone (k = 1).
@pytest.mark.parametrize("H,G,d,d_idx,k,S_lens,T_lens", [
    (32, 2, 128, 128, 8, [1100, 70], [180, 70]),
    (4, 1, 64, 64, 1, [334, 500], [166, 257]),
])
def test_kl_unit_other_shapes(exe, tmp_path, H, G, d, d_idx, k, S_lens, T_lens):
    _replay(exe, tmp_path, False, 33, H, G, d, d_idx, k, S_lens, T_lens)
