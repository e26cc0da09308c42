"""Pins of the selection-policy oracle (oracle/selection_policies.py) against
things other than itself (CPU only):

* brute force: every subset of the non-forced causal blocks of the right
  size is enumerated and the one whose blocks rank best under (score
  descending, index ascending) wins;
* the defaults (no sink, local block only) reproduce the pinned final rule
  (oracle.msa_oracle.index_topk) exactly, for any B_k;
* the FLOP-matched sliding-window baseline (one sink block, k-1 local blocks)
  is the window written out and ignores the scores;
* invariants: |sel| = min(k, nb), the forced blocks are always in, ids
  ascending and causal.
"""
import itertools

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from oracle import msa_oracle as O
from oracle import selection_policies as P


def _brute(S, k, n_sink, n_local):
    lb = len(S) - 1
    if lb + 1 <= k:
        return list(range(lb + 1))
    forced = {b for b in range(lb + 1) if b < n_sink or b > lb - n_local}
    free = [b for b in range(lb + 1) if b not in forced]
    m = k - len(forced)
    key = lambda b: (-(S[b] if not np.isnan(S[b]) else -np.inf), b)  # noqa: E731
    best = min(itertools.combinations(free, m), key=lambda c: sorted(key(b) for b in c))
    return sorted(forced | set(best))


@st.composite
def _case(draw):
    k = draw(st.integers(2, 6))
    n_sink = draw(st.integers(0, 2))
    n_local = draw(st.integers(1, max(1, k - n_sink)))
    if n_sink + n_local > k:
        n_sink = k - n_local
    nb = draw(st.integers(1, 11))
    scores = draw(st.lists(st.sampled_from([-2.0, -1.0, 0.0, 1.0, 2.0, float("nan"), float("-inf")]),
                           min_size=nb, max_size=nb))
    return k, n_sink, n_local, np.array(scores)


@settings(max_examples=300, deadline=None)
@given(_case())
def test_policy_matches_brute_force(case):
    k, n_sink, n_local, S = case
    got = P.select_blocks_policy(S, k, n_sink, n_local)
    assert got == _brute(S, k, n_sink, n_local)
    lb = len(S) - 1
    assert len(got) == min(k, lb + 1)
    assert set(P.forced_blocks(lb, n_sink, n_local)) <= set(got)
    assert got == sorted(set(got)) and all(0 <= b <= lb for b in got)


@settings(max_examples=100, deadline=None)
@given(st.integers(1, 40), st.integers(2, 8), st.integers(0, 2 ** 31 - 1))
def test_window_baseline_ignores_scores(nb, k, seed):
    S = np.random.default_rng(seed).standard_normal(nb)
    want = P.window_baseline(nb - 1, k)
    assert P.select_blocks_policy(S, k, 1, k - 1) == want
    assert P.select_blocks_policy(-S, k, 1, k - 1) == want
    assert len(want) == min(k, nb)


@pytest.mark.parametrize("B_k", [2, 3, 4, 8])
def test_defaults_reproduce_the_final_rule(B_k):
    rng = np.random.default_rng(B_k)
    lens = [37, 5, 60]
    T_lens = [37, 5, 21]
    cu_k = np.concatenate([[0], np.cumsum(lens)]).tolist()
    cu_q = np.concatenate([[0], np.cumsum(T_lens)]).tolist()
    q_idx = rng.integers(-2, 3, size=(cu_q[-1], 2, 3)).astype(np.float64)
    k_idx = rng.integers(-2, 3, size=(cu_k[-1], 3)).astype(np.float64)
    for k in (1, 3, 5):
        np.testing.assert_array_equal(P.index_topk_policy(q_idx, k_idx, cu_q, cu_k, k, B_k),
                                      O.index_topk(q_idx, k_idx, cu_q, cu_k, k, B_k))


def test_forced_sink_is_kept_and_rejected_budgets():
    S = np.array([-5.0, 3.0, 2.0, 1.0, 0.0, 4.0, -1.0])    # block 0 scores worst
    assert P.select_blocks_policy(S, 3) == [1, 5, 6]
    assert P.select_blocks_policy(S, 3, n_sink=1) == [0, 5, 6]
    assert P.select_blocks_policy(S, 4, n_sink=1, n_local=2) == [0, 1, 5, 6]
    with pytest.raises(ValueError):
        P.select_blocks_policy(S, 3, n_sink=2, n_local=2)
    with pytest.raises(ValueError):
        P.select_blocks_policy(S, 3, n_sink=0, n_local=0)
