"""The rounding of the tensor-core Main Branch backward against the fp64
oracle (oracle/main_backward.py), over more shapes than its GPU test covers.

The kernel (csrc/msa_attn_bwd_tc.cu) takes S and dP as fp32 sums of bf16
products, P = exp2(S sm_scale log2(e) - lse log2(e)) and dS = P (dP sm_scale -
D sm_scale) in fp32, with D = dO . O read from the forward's bf16 output, and
rounds P and dS to bf16 (round to nearest even) before the dV = P^T dO,
dK = dS^T Q and dQ = dS K products.  This model applies exactly those
roundings (the fp32 sums in a different order, which is below the bound's
scale) and checks that the GPU test's bound, 5e-3 x the largest |gradient|,
holds for every head group size, d, k and ragged lengths drawn; two planted
mistakes (D left out; dQ from P instead of dS) must break it."""
import numpy as np
import pytest
import torch

from oracle import main_backward as B
from oracle import msa_oracle as O

LOG2E = 1.4426950408889634


def _bf(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).bfloat16().double().numpy()


def _f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def _model(q, k, v, sel, dout, o_bf, lse, cu_q, cu_k, B_k, sm, mistake=None):
    T, H, d = q.shape
    G = k.shape[1]
    Hg = H // G
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    c = np.float32(sm * LOG2E)
    for b in range(len(cu_q) - 1):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
        for i, pos in enumerate(O.query_positions(q1 - q0, k1 - k0)):
            t = q0 + i
            for g in range(G):
                J = O.selected_token_set([int(x) for x in sel[t, g]], int(pos), B_k)
                Kj, Vj = k[k0 + J, g], v[k0 + J, g]
                for h in range(g * Hg, (g + 1) * Hg):
                    s = _f32(Kj @ q[t, h]).astype(np.float32)
                    l2 = np.float32(np.float32(lse[t, h]) * np.float32(LOG2E))
                    p = np.exp2(s * c - l2).astype(np.float64)
                    dp = _f32(Vj @ dout[t, h])
                    D = 0.0 if mistake == "no_D" else float(_f32(dout[t, h] @ o_bf[t, h]))
                    ds = _f32(p * _f32(dp * sm - np.float32(D * sm)))
                    pb, dsb = _bf(p), _bf(ds)
                    dq[t, h] = (pb if mistake == "dq_from_P" else dsb) @ Kj
                    dk[k0 + J, g] += np.outer(dsb, q[t, h])
                    dv[k0 + J, g] += np.outer(pb, dout[t, h])
    return dq, dk, dv


def _case(seed, H, G, d, k, S_lens, T_lens):
    B_k = 128
    rng = np.random.default_rng(seed)
    cu_k = np.concatenate([[0], np.cumsum(S_lens)]).astype(np.int64)
    cu_q = np.concatenate([[0], np.cumsum(T_lens)]).astype(np.int64)
    T, S = int(cu_q[-1]), int(cu_k[-1])
    q, kk, v = _bf(rng.standard_normal((T, H, d))), _bf(rng.standard_normal((S, G, d))), \
        _bf(rng.standard_normal((S, G, d)))
    dout = _bf(rng.standard_normal((T, H, d)))
    q_idx = rng.integers(-4, 5, size=(T, G, 32)).astype(np.float64)
    k_idx = rng.integers(-4, 5, size=(S, 32)).astype(np.float64)
    sel = O.index_topk(q_idx, k_idx, cu_q.tolist(), cu_k.tolist(), k, B_k)
    sm = d ** -0.5
    o, lse = O.msa_forward_rows(q, kk, v, sel, cu_q, cu_k, list(range(T)), B_k, sm)
    return dict(q=q, k=kk, v=v, sel=sel, dout=dout, o_bf=_bf(o), lse=lse, cu_q=cu_q, cu_k=cu_k, B_k=B_k, sm=sm)


def _errors(c, mistake=None):
    got = _model(c["q"], c["k"], c["v"], c["sel"], c["dout"], c["o_bf"], c["lse"], c["cu_q"], c["cu_k"], c["B_k"],
                 c["sm"], mistake)
    want = B.main_branch_backward(c["q"], c["k"], c["v"], c["sel"], c["dout"], c["cu_q"], c["cu_k"], c["B_k"], c["sm"])
    return [float(np.abs(a - w).max() / np.abs(w).max()) for a, w in zip(got, want)]


def _shapes():
    rng = np.random.default_rng(2024)
    out = []
    for n in range(12):
        G = int(rng.choice([1, 2]))
        Hg = int(rng.choice([4, 8, 16]))
        d = int(rng.choice([64, 128]))
        k = int(rng.choice([1, 3, 8]))
        S_lens = [int(x) for x in rng.integers(129, 700, size=2)]
        T_lens = [int(min(s, x)) for s, x in zip(S_lens, rng.integers(20, 90, size=2))]
        out.append((100 + n, Hg * G, G, d, k, S_lens, T_lens))
    return out


@pytest.mark.parametrize("seed,H,G,d,k,S_lens,T_lens", _shapes())
def test_bf16_p_and_ds_stay_within_the_gpu_bound(seed, H, G, d, k, S_lens, T_lens):
    errs = _errors(_case(seed, H, G, d, k, S_lens, T_lens))
    assert max(errs) < 5e-3, dict(zip(("dq", "dk", "dv"), errs))


@pytest.mark.parametrize("mistake", ["no_D", "dq_from_P"])
def test_planted_mistakes_break_the_bound(mistake):
    errs = _errors(_case(7, 16, 2, 64, 8, [600, 300], [80, 60]), mistake)
    assert max(errs) > 5e-3, (mistake, errs)
