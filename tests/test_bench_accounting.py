"""The bench's per-kernel work split (roofline.tile_split, vectorised with torch
sorting) against the planner's rule written out with plain loops: tiles of
UQ consecutive rows of a pass that lie in one sequence; a block chosen by at
least theta of a tile's queries (one group) is covered; a query whose every
selection is covered needs no combine."""
import numpy as np
import pytest
import torch

from oracle import msa_oracle as O
from block_sparse_long_exp_b200 import roofline as R


def _selection(lengths, G, k, seed):
    rng = np.random.default_rng(seed)
    S = sum(lengths)
    d_idx = 8
    q_idx = rng.integers(-2, 3, size=(S, G, d_idx)).astype(np.float64)
    k_idx = rng.integers(-2, 3, size=(S, d_idx)).astype(np.float64)
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + L)
    return O.index_topk(q_idx, k_idx, cu, cu, k, 128), cu


def _brute(sel, cu, H, G, d, theta, q_chunk):
    T, _, k = sel.shape
    Hg = H // G
    UQ = 2 * (128 // max(Hg, 8))
    qpt = UQ // 2
    seq_of = np.searchsorted(np.array(cu), np.arange(T), side="right") - 1
    pos = np.array([t - cu[seq_of[t]] for t in range(T)])     # prefill: S_b == T_b
    covered = np.zeros(sel.shape, dtype=bool)
    mma_tiles = 0
    rows = T if q_chunk <= 0 else q_chunk
    for t0 in range(0, T, rows):
        t1 = min(T, t0 + rows)
        for r0 in range(t0, t1, UQ):
            r1 = min(t1, r0 + UQ)
            if seq_of[r0] != seq_of[r1 - 1] or theta <= 0:
                continue
            for g in range(G):
                count = {}
                for t in range(r0, r1):
                    for b in sel[t, g]:
                        if b >= 0:
                            count[int(b)] = count.get(int(b), 0) + 1
                dense = {b for b, c in count.items() if c >= theta}
                mma_tiles += len(dense) * (2 if r1 - r0 > qpt else 1)
                for t in range(r0, r1):
                    for s in range(k):
                        covered[t, g, s] = sel[t, g, s] >= 0 and int(sel[t, g, s]) in dense
    tile = kv = 0
    merged = npairs = complete = 0
    for t in range(T):
        lb = pos[t] // 128
        for g in range(G):
            valid = sel[t, g] >= 0
            for s in range(k):
                if not valid[s]:
                    continue
                att = 128 if sel[t, g, s] < lb else pos[t] % 128 + 1
                if covered[t, g, s]:
                    tile += att
                else:
                    kv += att
            ncov = covered[t, g].sum()
            if ncov > 0 and ncov == valid.sum():
                complete += 1
            else:
                npairs += 1
                merged += (valid & ~covered[t, g]).sum() + (1 if ncov > 0 else 0)
    comb = merged * Hg * (d * 2 + 4) + npairs * 8 + npairs * (Hg * d * 2 + Hg * 4)
    return {"tile_flops": 4.0 * d * Hg * tile, "kv_flops": 4.0 * d * Hg * kv, "combine_bytes": float(comb),
            "combine_pairs": npairs, "complete_pairs": complete,
            "tile_mma_flops": float(mma_tiles * 4 * 128 * 128 * d)}


@pytest.mark.parametrize("H,G", [(64, 4), (8, 2)])
@pytest.mark.parametrize("theta,q_chunk", [(0, 0), (1, 0), (3, 0), (5, 0), (3, 300)])
def test_tile_split_matches_the_rule(H, G, theta, q_chunk):
    lengths = [1500, 130, 917]                    # up to 12 blocks, k = 4: real top-k choices
    sel, cu = _selection(lengths, G, k=4, seed=5)
    got = R.tile_split(torch.from_numpy(sel), cu, cu, H, G, 64, 128, theta, q_chunk)
    ref = _brute(sel, cu, H, G, 64, theta, q_chunk)
    for key, v in ref.items():
        assert got[key] == pytest.approx(v), key
    # the split never loses work: it always adds up to the method's main-branch FLOPs
    work = R.prefill_work(lengths, lengths, H, G, 64, 8, 128, 4)
    assert got["tile_flops"] + got["kv_flops"] == pytest.approx(work["main_flops"])


def test_code_hash_ignores_comments_and_layout_only():
    """roofline.traffic stays valid across comment edits, not across code edits."""
    import bench
    a = 'int x = 1; // note\n/* a\n block */ float y;\nconst char* s = "// kept";\nchar c = \'"\';\n'
    b = 'int x = 1;\n\n   float   y;   // other note\nconst char* s = "// kept";\nchar c = \'"\';\n'
    c = 'int x = 2; // note\n float y;\nconst char* s = "// kept";\nchar c = \'"\';\n'
    d = 'int x = 1;\n float y;\nconst char* s = "// kept!";\nchar c = \'"\';\n'
    T = bench.code_tokens
    assert T(a) == T(b)
    assert T(a) != T(c) and T(a) != T(d)          # code and string literals count
    assert "// kept" in T(a)


def test_recorded_traffic_matches_current_code():
    """Every entry of profiles/traffic.json names a kernel file that exists, and the
    bench reads its figure back exactly when the code hash matches."""
    import json
    import os
    import bench
    d = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    for name, e in d.items():
        sha = bench.kernel_source_sha(e["source"])
        assert sha is not None, name
        want = e["dram_bytes_per_launch"] if sha == e["source_sha"] else None
        assert bench.traffic_for(name) == want


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one JSON
    line with the contract's keys and the same config our arm prints."""
    import json
    import os
    import subprocess
    import sys
    import bench
    from block_sparse_long_exp_b200 import workloads as W
    root = bench.ROOT
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_n4096", "--steps", "2", "--warmup", "1"], capture_output=True, text=True,
                       timeout=600, cwd=root, env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    w = W.WORKLOADS["tiny_n4096"]
    args = bench.build_parser().parse_args(["--workload", "tiny_n4096"])
    assert line["config"] == bench.run_config(args, w, line["config"]["T"], 1)
    assert bench.pass_rows(-1, 131072) == 0 and bench.pass_rows(-1, 131073) == 131072
    assert bench.pass_rows(700, 5000) == 700


def test_training_leg_reports_each_kernel_against_its_peak():
    # the leg's plumbing, with stand-ins for the library calls that accept
    # exactly the arguments the real binding functions take
    import inspect
    import types

    import bench
    from block_sparse_long_exp_b200 import msa as M
    from block_sparse_long_exp_b200 import workloads as W

    w = W.WORKLOADS[bench.PREFILL]
    T = 300
    calls = []

    def stand_in(name, ret):
        sig = inspect.signature(getattr(M, name))

        def f(*a, **kw):
            sig.bind(*a, **kw)
            calls.append(name)
            return ret(*a, **kw)
        return f
    lib = types.SimpleNamespace(
        make_shape=M.make_shape,
        make_varlen=stand_in("make_varlen", lambda *a: None),
        msa_index_topk=stand_in("msa_index_topk", lambda *a, **kw: torch.zeros(T, w.G, w.k, dtype=torch.int32)),
        msa_sparse_attn_prefill=stand_in("msa_sparse_attn_prefill",
                                         lambda sh, sq, q, *a, **kw: (torch.zeros_like(q), torch.zeros(T, w.H))),
        msa_sparse_attn_backward=stand_in("msa_sparse_attn_backward", lambda *a, **kw: (None, None, None)),
        msa_index_kl=stand_in("msa_index_kl", lambda *a, **kw: (torch.zeros(T, w.G), torch.zeros(T, w.G))),
        msa_index_kl_backward=stand_in("msa_index_kl_backward", lambda *a, **kw: (None, None)),
        msa_profile_reset=stand_in("msa_profile_reset", lambda: None),
        msa_profile_enable=stand_in("msa_profile_enable", lambda on: None),
        msa_profile_read=stand_in("msa_profile_read", lambda name=None: (8.0, 4)))
    args = bench.build_parser().parse_args(["--training-T", str(T), "--training-steps", "4",
                                            "--training-warmup", "3"])
    assert args.training                         # the training leg is part of the default run
    sync = torch.cuda.synchronize
    torch.cuda.synchronize = lambda *a: None
    try:
        res = bench.training_leg(args, w, W, R, lib, torch, device="cpu")
    finally:
        torch.cuda.synchronize = sync
    # one checked pass, the warm-up, the timed passes, one checked pass
    assert calls.count("msa_sparse_attn_backward") == 1 + 3 + 4 + 1
    tw = R.training_work([T], [T], w.H, w.G, w.d, w.d_idx, w.B_k, w.k)
    assert res["T"] == T and res["peak"] == R.alu_fp32_tflops()
    kr = res["kernels"]["index_kl_grad"]
    assert kr["bound"] == "alu" and kr["ms_per_launch"] == 2.0 and kr["flops_per_launch"] == tw["kl_grad_alu_flops"]
    assert kr["achieved"] == pytest.approx(tw["kl_grad_alu_flops"] / 2e-3 / 1e12)
    assert kr["frac"] == pytest.approx(kr["achieved"] / R.alu_fp32_tflops())
    # the backward against the measured bf16 burst peak
    kr = res["kernels"]["attn_bwd"]
    assert kr["bound"] == "tensor" and kr["flops_per_launch"] == tw["backward_flops"]
    assert kr["achieved"] == pytest.approx(tw["backward_flops"] / 2e-3 / 1e12)
    assert kr["frac"] == pytest.approx(kr["achieved"] / bench.load_peaks()[0]["bf16_tflops"])
    # the gradient's CUDA-core share: dq_idx and dk_idx, 2 d_idx FLOPs each per (query, group, key)
    assert tw["kl_grad_alu_flops"] == pytest.approx(tw["pairs"] * 4 * w.G * w.d_idx)
    assert tw["kl_tensor_flops"] + tw["kl_grad_alu_flops"] == pytest.approx(tw["kl_grad_flops"])
    assert res["kernels"]["index_kl_grad"]["tensor"]["flops_per_launch"] == tw["kl_tensor_flops"]
    # the KL target against the exponential rate: one exp per head and pair
    kr = res["kernels"]["index_kl"]
    assert kr["bound"] == "mufu" and kr["ms_per_launch"] == 2.0
    assert tw["kl_exps"] == pytest.approx(tw["pairs"] * w.H)
    assert R.mufu_gexps() == pytest.approx(148 * 16 * 1.965)
    assert kr["achieved"] == pytest.approx(tw["kl_exps"] / 2e-3 / 1e9)
    assert kr["frac"] == pytest.approx(kr["achieved"] / R.mufu_gexps())
    assert kr["tensor"]["achieved"] == pytest.approx(tw["pairs"] * (2 * w.H * w.d + 2 * w.G * w.d_idx) / 2e-3 / 1e12)
    assert tw["kl_tensor_flops"] == pytest.approx(tw["kl_flops"])   # both products of the target
    assert kr["tensor"]["frac"] == pytest.approx(kr["tensor"]["achieved"] / kr["tensor"]["peak"])
