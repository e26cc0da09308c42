"""The FMA-pipe exponential of the attention kernels (msa_exp2.cuh): its host
build (bit-identical to the device one: plain fp32 with explicitly rounded
operations) is compared with exp2 in double precision over ~39M inputs, and
its coefficients are checked to be the committed Remez fit rounded to fp32."""
import os
import re
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_long_exp_b200", "csrc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_exp2_fma_error_bound(tmp_path):
    exe = str(tmp_path / "exp2_host")
    subprocess.run(["g++", "-O2", "-std=c++17", "-ffp-contract=off", "-Wall", "-Werror", f"-I{CSRC}",
                    os.path.join(ROOT, "tests", "c", "exp2_host.cc"), "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    worst = float(re.search(r"largest relative error ([0-9.e+-]+)", r.stdout).group(1))
    assert worst <= 7.6e-5                      # far below bf16's half ulp, 2^-9


def test_exp2_coefficients_are_the_fit():
    sys.path.insert(0, CSRC)
    try:
        import exp2_poly_fit as F
    finally:
        sys.path.remove(CSRC)
    import numpy as np
    c32 = F.remez(3).astype(np.float32)
    text = open(os.path.join(CSRC, "msa_exp2.cuh")).read()
    lits = re.search(r"c0 = (\S+)f, c1 = (\S+)f, c2 = (\S+)f, c3 = (\S+)f;", text).groups()
    assert [float.fromhex(v) for v in lits] == [float(c) for c in c32]
    assert F.fp32_horner_error(c32) < 7.6e-5
