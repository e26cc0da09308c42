"""Pins of the fp64 oracle against things other than itself (CPU only).

* a hand-worked example (tests/golden/hand_selection.json);
* brute force on tiny inputs: token scores by explicit loops, block maxima by
  Python max, the selection by enumerating every subset;
* the exp-free claim: ranking blocks by max-pooled softmax probabilities picks
  the same blocks as ranking by raw scores;
* the special case k >= number of causal blocks, which is dense causal GQA,
  computed by torch's scaled_dot_product_attention in fp64;
* the general sparse case against scaled_dot_product_attention with an explicit
  per-group token mask built from the selection by plain loops;
* the log-sum-exp combine against the softmax over the union;
* the reverse index against a round trip.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import msa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_selection.json")


# ---------------------------------------------------------------- golden ----

def test_golden_hand_selection():
    fx = json.load(open(GOLDEN))
    st = fx["setup"]
    S, G, B_k, k = st["S"], st["G"], st["B_k"], st["k"]
    k_idx = np.stack([st["k_idx_col0"], st["k_idx_col1"]], axis=1).astype(np.float64)
    q_idx = np.tile(np.asarray(st["q_idx_every_query"], np.float64)[None], (S, 1, 1))
    sel = O.index_topk(q_idx, k_idx, [0, S], [0, S], k, B_k)
    Kz = np.zeros((S, G, 2))
    V = np.zeros((S, G, 2))
    V[:, :, 0] = np.arange(S)[:, None]
    V[:, :, 1] = 1.0
    Q = np.ones((S, st["H"], 2))
    for case in fx["cases"]:
        t = case["t"]
        assert sel[t].tolist() == case["sel"], case["why"]
        if "o_g0" in case:
            o, lse = O.msa_forward_rows(Q, Kz, V, sel, [0, S], [0, S], [t], B_k, 1.0)
            np.testing.assert_allclose(o[0, 0], case["o_g0"], rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[0, 0], math.log(case["lse_g0_tokens"]),
                                       rtol=0, atol=1e-12)
            if "o_g1" in case:
                np.testing.assert_allclose(o[0, 1], case["o_g1"], rtol=0, atol=1e-12)
                np.testing.assert_allclose(lse[0, 1], math.log(case["lse_g1_tokens"]),
                                           rtol=0, atol=1e-12)


# ----------------------------------------------------------- brute force ----

def _brute_select(q_row, k_rows, pos, B_k, k):
    """Selection by explicit loops and subset enumeration."""
    scores = []
    for j in range(pos + 1):
        acc = 0.0
        for c in range(len(q_row)):
            acc += float(q_row[c]) * float(k_rows[j][c])
        scores.append(acc)
    lb = pos // B_k
    bmax = []
    for b in range(lb + 1):
        vals = [scores[j] for j in range(b * B_k, min((b + 1) * B_k, pos + 1))]
        bmax.append(max(vals))
    if lb + 1 <= k:
        return list(range(lb + 1))

    def beats(a, b):  # a ranks above b: higher score, ties to the lower index
        return bmax[a] > bmax[b] or (bmax[a] == bmax[b] and a < b)

    found = []
    for subset in itertools.combinations(range(lb), k - 1):
        rest = [b for b in range(lb) if b not in subset]
        if all(beats(a, b) for a in subset for b in rest):
            found.append(list(subset))
    assert len(found) == 1, "the ranking is a total order: exactly one top set"
    return sorted(found[0]) + [lb]


@pytest.mark.parametrize("seed", range(6))
def test_selection_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    B_k = int(rng.integers(2, 5))
    k = int(rng.integers(2, 5))
    nb = int(rng.integers(k + 1, 11))
    S = nb * B_k - int(rng.integers(0, B_k))       # ragged last block
    G, d_idx = 2, 3
    # small integers so that ties are frequent
    q_idx = rng.integers(-2, 3, size=(S, G, d_idx)).astype(np.float64)
    k_idx = rng.integers(-2, 3, size=(S, d_idx)).astype(np.float64)
    sel = O.index_topk(q_idx, k_idx, [0, S], [0, S], k, B_k)
    for t in range(S):
        for g in range(G):
            want = _brute_select(q_idx[t, g], k_idx, t, B_k, k)
            got = [int(x) for x in sel[t, g] if x >= 0]
            assert got == want, (t, g)
            assert all(x == -1 for x in sel[t, g][len(want):])


def test_selection_chunked_and_varlen_positions():
    """Queries are the last T_b tokens of each sequence; check against brute
    force with explicit positions."""
    rng = np.random.default_rng(11)
    B_k, k, G, d_idx = 3, 3, 1, 2
    S_lens = [17, 5, 12]
    T_lens = [6, 5, 1]
    cu_k = np.concatenate([[0], np.cumsum(S_lens)])
    cu_q = np.concatenate([[0], np.cumsum(T_lens)])
    k_idx = rng.integers(-2, 3, size=(cu_k[-1], d_idx)).astype(np.float64)
    q_idx = rng.integers(-2, 3, size=(cu_q[-1], G, d_idx)).astype(np.float64)
    sel = O.index_topk(q_idx, k_idx, cu_q, cu_k, k, B_k)
    for b in range(3):
        for i in range(T_lens[b]):
            t = cu_q[b] + i
            pos = S_lens[b] - T_lens[b] + i
            want = _brute_select(q_idx[t, 0], k_idx[cu_k[b]:cu_k[b + 1]], pos, B_k, k)
            assert [int(x) for x in sel[t, 0] if x >= 0] == want


def test_nan_scores_rank_last_but_fill_slots():
    B_k, k = 2, 3
    s = np.array([np.nan, np.nan, 1.0, 0.0, np.nan, np.nan, -np.inf, -np.inf, 5.0, 5.0])
    S = O.block_max_pool(s, B_k)
    assert S[0] == -np.inf and S[1] == 1.0 and S[2] == -np.inf and S[3] == -np.inf
    # candidates 0..3, scores [-inf, 1, -inf, -inf]: block 1, then the tie of the
    # -inf blocks goes to the lowest index (0); local block 4 is forced
    assert O.select_blocks(S, k) == [0, 1, 4]


# -------------------------------------------------------------- exp-free ----

@pytest.mark.parametrize("hot", [False, True])
def test_exp_free_ranking_equals_softmax_ranking(hot):
    """Selecting on raw scores equals selecting on max-pooled softmax weights
    (the exp-free claim).  The softmax is ranked in log form (s/sqrt(d_idx) -
    LSE), an exact monotone shift, so that underflow cannot create ties; rows
    where exp does not underflow are also checked in the exp form."""
    rng = np.random.default_rng(5)
    B_k, k, d_idx, S = 8, 4, 16, 200
    k_idx = rng.integers(-4, 5, size=(S, d_idx)).astype(np.float64)
    if hot:
        for b in (3, 11, 17):
            k_idx[b * B_k:(b + 1) * B_k] *= 3
    q_idx = rng.integers(-4, 5, size=(S, 1, d_idx)).astype(np.float64)
    sel = O.index_topk(q_idx, k_idx, [0, S], [0, S], k, B_k)
    checked_exp = 0
    for t in range(S):
        s = O.index_scores(q_idx[t, 0], k_idx, t)
        z = s / math.sqrt(d_idx)
        m = z.max()
        logp = z - (m + math.log(np.exp(z - m).sum()))
        chosen = O.select_blocks(O.block_max_pool(logp, B_k), k)
        assert chosen == [int(x) for x in sel[t, 0] if x >= 0]
        p = np.exp(logp)
        if np.all(p > 0):
            checked_exp += 1
            assert O.select_blocks(O.block_max_pool(p, B_k), k) == chosen
    assert checked_exp > 50


# ------------------------------------------------------ dense equivalence ----

def _sdpa(q, k, v, mask, scale):
    """torch fp64 scaled_dot_product_attention; q [T,H,d], k/v [S,G,d] (GQA),
    mask [H or 1, T, S] bool (True = attend)."""
    H, G = q.shape[1], k.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(k).permute(1, 0, 2)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2)[None]
    m = torch.from_numpy(mask)[None]
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=m, scale=scale, enable_gqa=(H != G))
    return o[0].permute(1, 0, 2).numpy()


def test_dense_special_case_equals_causal_gqa():
    """k >= number of causal blocks: MSA is dense causal GQA attention."""
    rng = np.random.default_rng(3)
    T = S = 45
    H, G, d, d_idx, B_k = 4, 2, 8, 4, 8
    k = 6                                  # nb = 6 <= k
    q = rng.standard_normal((T, H, d))
    kk = rng.standard_normal((S, G, d))
    v = rng.standard_normal((S, G, d))
    q_idx = rng.integers(-4, 5, size=(T, G, d_idx)).astype(np.float64)
    k_idx = rng.integers(-4, 5, size=(S, d_idx)).astype(np.float64)
    sel = O.index_topk(q_idx, k_idx, [0, T], [0, S], k, B_k)
    scale = 1 / math.sqrt(d)
    o, _ = O.msa_forward_rows(q, kk, v, sel, [0, T], [0, S], list(range(T)), B_k, scale)
    causal = np.tril(np.ones((T, S), dtype=bool))[None]
    ref = _sdpa(q, kk, v, causal, scale)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_sparse_case_equals_masked_attention():
    """General selection: equals SDPA with the per-group mask 'token j lies in a
    selected block of (t, g) and j <= t', the mask built by plain loops."""
    rng = np.random.default_rng(4)
    T = S = 70
    H, G, d, d_idx, B_k, k = 4, 2, 8, 4, 8, 3
    q = rng.standard_normal((T, H, d))
    kk = rng.standard_normal((S, G, d))
    v = rng.standard_normal((S, G, d))
    q_idx = rng.integers(-4, 5, size=(T, G, d_idx)).astype(np.float64)
    k_idx = rng.integers(-4, 5, size=(S, d_idx)).astype(np.float64)
    sel = O.index_topk(q_idx, k_idx, [0, T], [0, S], k, B_k)
    mask = np.zeros((H, T, S), dtype=bool)
    for h in range(H):
        g = h // (H // G)
        for t in range(T):
            for j in range(t + 1):
                if (j // B_k) in set(int(x) for x in sel[t, g]):
                    mask[h, t, j] = True
    scale = 1 / math.sqrt(d)
    o, lse = O.msa_forward_rows(q, kk, v, sel, [0, T], [0, S], list(range(T)), B_k, scale)
    ref = _sdpa(q, kk, v, mask, scale)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    # lse against its definition over the masked logits
    for t in (0, 17, 69):
        for h in range(H):
            g = h // (H // G)
            lg = scale * (kk[:, g] @ q[t, h])
            want = np.log(np.sum(np.exp(lg[mask[h, t]])))
            assert abs(lse[t, h] - want) < 1e-12


def test_decode_positions_equal_last_prefill_row():
    """Decode (one query at position L-1) equals the last row of a prefill."""
    rng = np.random.default_rng(9)
    S, H, G, d, d_idx, B_k, k = 50, 2, 1, 4, 3, 4, 3
    q = rng.standard_normal((S, H, d))
    kk = rng.standard_normal((S, G, d))
    v = rng.standard_normal((S, G, d))
    q_idx = rng.integers(-4, 5, size=(S, G, d_idx)).astype(np.float64)
    k_idx = rng.integers(-4, 5, size=(S, d_idx)).astype(np.float64)
    sel_p = O.index_topk(q_idx, k_idx, [0, S], [0, S], k, B_k)
    sel_d = O.index_topk(q_idx[-1:], k_idx, [0, 1], [0, S], k, B_k)
    assert sel_d[0].tolist() == sel_p[-1].tolist()
    o_p, _ = O.msa_forward_rows(q, kk, v, sel_p, [0, S], [0, S], [S - 1], B_k, 0.5)
    o_d, _ = O.msa_forward_rows(q[-1:], kk, v, sel_d, [0, 1], [0, S], [0], B_k, 0.5)
    np.testing.assert_allclose(o_d, o_p, rtol=0, atol=1e-14)


# ---------------------------------------------------------------- combine ----

def test_lse_combine_equals_union_softmax():
    rng = np.random.default_rng(7)
    B_k, d, Hg = 4, 5, 3
    S = 40
    q = rng.standard_normal((Hg, d))
    K = rng.standard_normal((S, d)) * 2
    V = rng.standard_normal((S, d))
    blocks = [1, 4, 6, 9]
    pos = 38
    full_o, full_lse = O.main_branch(q, K, V, blocks, pos, B_k, 0.7)
    parts = [O.main_branch(q, K, V, [b], pos, B_k, 0.7) for b in blocks]
    o, lse = O.lse_combine([p[0] for p in parts], [p[1] for p in parts])
    np.testing.assert_allclose(o, full_o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, full_lse, rtol=0, atol=1e-13)


def test_lse_combine_closed_form_two_parts():
    # two partials with equal lse get equal weight 1/2; lse grows by log 2
    o, lse = O.lse_combine(np.array([[2.0, 0.0], [0.0, 4.0]]), np.array([1.5, 1.5]))
    np.testing.assert_allclose(o, [1.0, 2.0], atol=1e-15)
    assert abs(lse - (1.5 + math.log(2))) < 1e-15


# ----------------------------------------------------------- reverse index ----

def test_invert_selection_round_trip():
    rng = np.random.default_rng(8)
    B_k, k = 4, 3
    S_lens = [30, 9, 21]
    cu = np.concatenate([[0], np.cumsum(S_lens)])
    G, d_idx = 2, 3
    q_idx = rng.integers(-3, 4, size=(cu[-1], G, d_idx)).astype(np.float64)
    k_idx = rng.integers(-3, 4, size=(cu[-1], d_idx)).astype(np.float64)
    sel = O.index_topk(q_idx, k_idx, cu, cu, k, B_k)
    lists = O.invert_selection(sel, cu, cu, B_k)
    rebuilt = {}
    total = 0
    for (b, g, blk), ts in lists.items():
        assert ts == sorted(ts) and len(set(ts)) == len(ts)
        for t in ts:
            assert cu[b] <= t < cu[b + 1]
            rebuilt.setdefault((t, g), []).append(blk)
            total += 1
    assert total == int(np.sum(sel >= 0))
    for t in range(cu[-1]):
        for g in range(G):
            want = [int(x) for x in sel[t, g] if x >= 0]
            assert sorted(rebuilt[(t, g)]) == want


# -------------------------------------------------- randomised properties ----

from hypothesis import given, settings, strategies as st  # noqa: E402


@st.composite
def _tiny_layer(draw):
    G = draw(st.sampled_from([1, 2]))
    Hg = draw(st.sampled_from([1, 2]))
    B_k = draw(st.sampled_from([3, 4]))
    k = draw(st.integers(1, 5))
    nseq = draw(st.integers(1, 3))
    S_lens = [draw(st.integers(1, 24)) for _ in range(nseq)]
    T_lens = [draw(st.integers(0, S)) for S in S_lens]
    seed = draw(st.integers(0, 2 ** 31 - 1))
    return G, Hg, B_k, k, S_lens, T_lens, seed


@settings(max_examples=60, deadline=None)
@given(_tiny_layer())
def test_random_layers_match_brute_force_and_masked_sdpa(layer):
    """Random varlen layers (queries are the last T_b tokens): the selection
    equals subset enumeration, the output equals fp64 SDPA with a token mask
    built by loops, sequence by sequence."""
    G, Hg, B_k, k, S_lens, T_lens, seed = layer
    rng = np.random.default_rng(seed)
    H, d, d_idx = G * Hg, 4, 3
    S, T = sum(S_lens), sum(T_lens)
    cu_k = np.concatenate([[0], np.cumsum(S_lens)]).tolist()
    cu_q = np.concatenate([[0], np.cumsum(T_lens)]).tolist()
    q = rng.standard_normal((T, H, d))
    kk = rng.standard_normal((S, G, d))
    v = rng.standard_normal((S, G, d))
    q_idx = rng.integers(-2, 3, size=(T, G, d_idx)).astype(np.float64)
    k_idx = rng.integers(-2, 3, size=(S, d_idx)).astype(np.float64)
    sel = O.index_topk(q_idx, k_idx, cu_q, cu_k, k, B_k)
    scale = 1 / math.sqrt(d)
    o, _ = O.msa_forward_rows(q, kk, v, sel, cu_q, cu_k, list(range(T)), B_k, scale)
    for b in range(len(S_lens)):
        Tb, Sb = T_lens[b], S_lens[b]
        if Tb == 0:
            continue
        ks = k_idx[cu_k[b]:cu_k[b + 1]]
        mask = np.zeros((H, Tb, Sb), dtype=bool)
        for i in range(Tb):
            t, pos = cu_q[b] + i, Sb - Tb + i
            for g in range(G):
                want = _brute_select(q_idx[t, g], ks, pos, B_k, k)
                got = [int(x) for x in sel[t, g] if x >= 0]
                assert got == want, (b, i, g)
                for h in range(g * Hg, (g + 1) * Hg):
                    for j in range(pos + 1):
                        mask[h, i, j] = (j // B_k) in want
        # SDPA over this sequence's queries and keys
        qb = q[cu_q[b]:cu_q[b + 1]]
        ref = _sdpa(qb, kk[cu_k[b]:cu_k[b + 1]], v[cu_k[b]:cu_k[b + 1]], mask, scale)
        np.testing.assert_allclose(o[cu_q[b]:cu_q[b + 1]], ref, rtol=0, atol=1e-12)


def _brute_top_set(S, lb, k):
    """Subset enumeration: the one (k-1)-subset of blocks 0..lb-1 whose every
    member beats every non-member (higher score, ties to the lower index; NaN
    as -inf), plus the local block lb; all blocks when lb + 1 <= k."""
    if lb + 1 <= k:
        return list(range(lb + 1))
    sc = [(-np.inf if np.isnan(x) else float(x)) for x in S]

    def beats(a, b):
        return sc[a] > sc[b] or (sc[a] == sc[b] and a < b)

    for subset in itertools.combinations(range(lb), k - 1):
        rest = [b for b in range(lb) if b not in subset]
        if all(beats(a, b) for a in subset for b in rest):
            return sorted(subset) + [lb]
    raise AssertionError("no top set")


@pytest.mark.parametrize("seed", range(4))
def test_key_range_candidates_merge_to_the_selection(seed):
    """A decode cache cut into key ranges: each range's first k-1 blocks
    (block_candidates), made global and merged (merge_block_candidates), give
    the selection of the whole cache: equal to select_blocks and, on small
    cases, to subset enumeration.  Integer scores (many ties) and NaNs; the
    ranges are random cuts of the non-local blocks."""
    rng = np.random.default_rng(100 + seed)
    for _ in range(400):
        nb = int(rng.integers(1, 30))
        k = int(rng.integers(1, 8))
        S = rng.integers(-3, 4, size=nb).astype(np.float64)
        S[rng.random(nb) < 0.08] = np.nan
        lb = nb - 1
        ncut = int(rng.integers(0, min(4, max(lb, 1))))
        cuts = sorted(rng.choice(np.arange(1, lb), size=ncut, replace=False).tolist()) if lb > 1 else []
        bounds = [0] + cuts + [lb]
        ids, scores = [], []
        for a, b in zip(bounds[:-1], bounds[1:]):
            ci, cs = O.block_candidates(S[a:b], k)
            assert len(ci) == min(k - 1, b - a)
            ids += [a + i for i in ci]
            scores += cs
        got = O.merge_block_candidates(ids, scores, lb, k)
        assert got == O.select_blocks(S, k)
        if lb <= 10:
            assert got == _brute_top_set(S, lb, k)


def test_key_range_candidates_catch_planted_mistakes():
    """Ties broken toward the higher index, or NaN ranked above numbers, in
    either function change the merged selection on some cut."""
    rng = np.random.default_rng(7)

    def cand_high_tie(S, k):
        keys = np.where(np.isnan(S), -np.inf, S)
        order = np.lexsort((-np.arange(len(keys)), -keys))[: k - 1]
        return [int(b) for b in order], [float(keys[b]) for b in order]

    def cand_nan_high(S, k):
        keys = np.where(np.isnan(S), np.inf, S)
        order = np.lexsort((np.arange(len(keys)), -keys))[: k - 1]
        return [int(b) for b in order], [float(keys[b]) for b in order]

    for bad in (cand_high_tie, cand_nan_high):
        caught = False
        for _ in range(300):
            nb, k = int(rng.integers(6, 20)), int(rng.integers(2, 5))
            S = rng.integers(-2, 3, size=nb).astype(np.float64)
            S[rng.random(nb) < 0.1] = np.nan
            lb = nb - 1
            mid = int(rng.integers(1, lb))
            ids, scores = [], []
            for a, b in ((0, mid), (mid, lb)):
                ci, cs = bad(S[a:b], k)
                ids += [a + i for i in ci]
                scores += cs
            if O.merge_block_candidates(ids, scores, lb, k) != O.select_blocks(S, k):
                caught = True
                break
        assert caught, bad.__name__
