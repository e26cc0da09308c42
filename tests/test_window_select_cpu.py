"""The sliding-window baseline's selection rule as the kernel runs it
(msa_window.h, built for the host with g++) against the selection-policy
oracle (oracle/selection_policies.py): with n_sink sink blocks and k - n_sink
local ones every slot is forced, so the oracle's general rule must return the
same blocks for any scores; with one sink block it is the oracle's written-out
window.  Plus the entry point's host checks."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import selection_policies as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_long_exp_b200", "csrc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_window_rule_matches_the_oracle(tmp_path):
    exe = str(tmp_path / "window_host")
    subprocess.run(["g++", "-O2", "-std=c++17", "-Wall", "-Werror", f"-I{CSRC}",
                    os.path.join(ROOT, "tests", "c", "window_host.cc"), "-o", exe], check=True)
    lines = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.splitlines()
    rng = np.random.default_rng(3)
    assert len(lines) == 70 * sum(range(1, 10))
    for line in lines:
        v = [int(x) for x in line.split()]
        lb, k, n_sink, blocks = v[0], v[1], v[2], v[3:]
        got = [b for b in blocks if b >= 0]
        assert blocks[len(got):] == [-1] * (k - len(got))
        S = rng.standard_normal(lb + 1)
        assert got == P.select_blocks_policy(S, k, n_sink, k - n_sink), line
        if n_sink == 1:
            assert got == P.window_baseline(lb, k), line


def test_window_entry_point_host_checks():
    from block_sparse_long_exp_b200 import build, msa
    build.build()
    lib = msa.load_library()
    shape = msa.make_shape(64, 4, 128, 64, 16)
    cu = (ctypes.c_int32 * 2)(0, 0)
    seqs = msa.Varlen(1, 300, 300, 0, 300, 300, ctypes.addressof(cu), ctypes.addressof(cu))
    assert lib.msa_select_window(ctypes.byref(shape), ctypes.byref(seqs), 16, 256, 256, 1 << 20, None) == 1
    assert lib.msa_select_window(ctypes.byref(shape), ctypes.byref(seqs), -1, 256, 256, 1 << 20, None) == 1
    assert lib.msa_select_window(ctypes.byref(shape), ctypes.byref(seqs), 1, None, 256, 1 << 20, None) == 1
    assert lib.msa_select_window(ctypes.byref(shape), ctypes.byref(seqs), 1, 256, 256, 16, None) == 3
