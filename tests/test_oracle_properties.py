"""Property sweeps (hypothesis) over the CPU oracle on tiny inputs.

Each property is fixed by the mathematics, not by the oracle's own code: the
exact top-n selection against brute force over all subsets, the Quest score
as an upper bound of every head's block-maximum dot product (tight on
one-token blocks), and the split-KV merge against one pass over the whole
selection.
"""
from __future__ import annotations

import itertools

import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle as O
from block_sparse_gqa_min_b200 import workloads as W
from tests.helpers import bf16_to_f64, gather_tokens, make_case, oracle_cache, small_workload

SWEEP = settings(max_examples=40, deadline=None, suppress_health_check=[HealthCheck.too_slow])


def _brute_select(scores, n, L):
    """The n - L non-local blocks whose score sum is largest (lowest indices among
    equal sums), plus the L local blocks, ascending."""
    N = len(scores)
    best = None
    for sub in itertools.combinations(range(N - L), n - L):
        key = (sum(scores[list(sub)]) if sub else 0.0, [-x for x in sub])
        if best is None or key > best[0]:
            best = (key, sub)
    return sorted(list(best[1]) + list(range(N - L, N)))


@SWEEP
@given(scores=st.lists(st.integers(-3, 3), min_size=1, max_size=10), L=st.integers(0, 3),
       n_budget=st.integers(0, 12), n_min=st.integers(0, 4), tail=st.integers(0, 3))
def test_selection_is_best_subset(scores, L, n_budget, n_min, tail):
    """Integer scores (many ties): the selection maximises the score sum with the
    lowest-index tie-break, always holds the local blocks, and has n_eff blocks."""
    b = 4
    N = len(scores)
    sc = np.array(scores, dtype=np.float64)
    length = N * b - tail  # a partial last block changes nothing about the blocks
    idx, cnt = O.select(sc.reshape(1, 1, N), np.array([length], np.int32), b, n_budget, L, n_min)
    got = list(idx[0, 0, : cnt[0, 0]])
    n = O.num_selected(N, n_budget, L, n_min)
    assert n == min(N, max(min(L, N), n_min, n_budget))
    assert got == _brute_select(sc, n, min(L, N))


@SWEEP
@given(seed=st.integers(0, 10_000), b=st.sampled_from([1, 2, 4]), d=st.sampled_from([4, 8]),
       G=st.sampled_from([1, 2, 3]), nblk=st.integers(1, 6))
def test_quest_score_bounds_every_token(seed, b, d, G, nblk):
    """Quest score of block j >= sum over the group's heads of max_t q_h . k_t
    (products of bf16 values are exact in fp64), with equality on one-token
    blocks of a one-head group."""
    w = small_workload(H_q=2 * G, H_kv=2, d=d, b=b, len_lo=nblk * b, len_hi=nblk * b, n_budget=1, n_local=0)
    lay, li = make_case(w, seed=seed)
    c = oracle_cache(w, lay, li)
    sc = O.quest_scores(c, W.bf16_bits(li.q))
    qv = bf16_to_f64(W.bf16_bits(li.q))[0]
    for h in range(2):
        keys = gather_tokens(c, 0, h)
        for j in range(nblk):
            blk = keys[j * b:(j + 1) * b]
            bound = sum((blk @ qv[h * G + i]).max() for i in range(G))
            assert sc[0, h, j] >= bound - 1e-12 * (1 + abs(bound))
            if b == 1 and G == 1:
                assert sc[0, h, j] == pytest.approx(bound, rel=1e-12, abs=1e-12)


@SWEEP
@given(seed=st.integers(0, 10_000), S=st.integers(1, 5), n_budget=st.integers(1, 8),
       length=st.integers(1, 40))
def test_split_merge_equals_one_pass(seed, S, n_budget, length):
    """Attention over any partition of the selection into S splits, merged by
    LSE, equals one pass over the whole selection (empty splits included)."""
    w = small_workload(H_q=4, H_kv=2, d=8, b=4, len_lo=length, len_hi=length, n_budget=n_budget, n_local=1)
    lay, li = make_case(w, seed=seed)
    c = oracle_cache(w, lay, li)
    q = W.bf16_bits(li.q)
    full = O.decode(c, q, scale=w.scale, n_budget=n_budget, n_local=1, n_min=0)
    rng = np.random.default_rng(seed)
    o_part = np.zeros((1, w.H_q, S, w.d))
    l_part = np.full((1, w.H_q, S), -np.inf)
    for h in range(w.H_kv):
        cnt = int(full.sel_cnt[0, h])
        cuts = np.sort(rng.integers(0, cnt + 1, size=S - 1))
        bounds = [0, *cuts.tolist(), cnt]
        for sp in range(S):
            sub = full.sel_idx[0, h, bounds[sp]:bounds[sp + 1]]
            idx = np.zeros((1, w.H_kv, max(1, len(sub))), np.int32)
            cn = np.zeros((1, w.H_kv), np.int32)
            idx[0, h, : len(sub)] = sub
            cn[0, h] = len(sub)
            o, l = O.attend(c, q, idx, cn, w.scale)
            for qh in range(h * w.G, (h + 1) * w.G):
                o_part[0, qh, sp] = o[0, qh]
                l_part[0, qh, sp] = l[0, qh]
    out, lse = O.combine(o_part, l_part)
    np.testing.assert_allclose(out, full.out, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, full.lse, rtol=1e-12, atol=1e-12)
