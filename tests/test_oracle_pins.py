"""Pins of the CPU oracle against what the pages and mathematics fix.

No page prints a worked numeric example, so each pin is a hand-derived worked
example (tests/golden), a closed form, an invariant, a textbook or library
routine on a special case, or brute force on tiny inputs.  Each is chosen so a
plausible slip in the oracle (a dropped term, a wrong sign or index, min and
max swapped, a transposed operand) fails at least one of them.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_gqa_min_b200 import workloads as W
from tests.helpers import bf16_to_f64, gather_tokens, make_case, oracle_cache, small_workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(x) -> np.ndarray:
    return W.bf16_bits(torch.tensor(x, dtype=torch.float32).to(torch.bfloat16))


# --------------------------------------------------------------------------
# Hand-derived worked example
# --------------------------------------------------------------------------

def _golden_cache():
    g = json.load(open(os.path.join(GOLDEN, "quest_worked_example.json")))
    d, b = g["d"], g["b"]
    keys = np.array(g["keys"], dtype=np.float32)
    vals = np.array(g["values"], dtype=np.float32)
    nb = len(keys) // b
    k = _bits(keys.reshape(nb, 1, b, d))
    v = _bits(vals.reshape(nb, 1, b, d))
    c = O.Cache(k, v, None, np.array([g["len"]], np.int32), H_q=g["H_q"], max_blocks=nb)
    q = _bits(np.array(g["q"], dtype=np.float32).reshape(1, g["H_q"], d))
    return g, c, q


def test_golden_descriptors_scores_selection():
    g, c, q = _golden_cache()
    e = g["expected"]
    mn, mx = O.quest_desc(c)
    assert np.array_equal(mn[0, :, 0, :], np.array(e["desc_min"], float))
    assert np.array_equal(mx[0, :, 0, :], np.array(e["desc_max"], float))
    sc = O.quest_scores(c, q)
    assert np.array_equal(sc[0, 0], np.array(e["group_score"], float))
    idx, cnt = O.select(sc, c.seq_lens, c.b, g["n_budget"], g["n_local"], g["n_min"])
    assert list(idx[0, 0, : cnt[0, 0]]) == e["selected"]


def test_golden_attention_closed_form():
    g, c, q = _golden_cache()
    e = g["expected"]
    d = O.decode(c, q, scale=g["scale"], n_budget=g["n_budget"], n_local=g["n_local"], n_min=g["n_min"])
    vals = np.array(g["values"], float)[[0, 1, 4]]
    for h, key in enumerate(["logits_head0", "logits_head1"]):
        l = np.array(e[key], float)
        w = np.exp(l) / np.exp(l).sum()
        np.testing.assert_allclose(d.out[0, h], w @ vals, rtol=0, atol=1e-14)
        np.testing.assert_allclose(d.lse[0, h], math.log(np.exp(l).sum()), rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# Descriptors
# --------------------------------------------------------------------------

@pytest.mark.parametrize("paged", [False, True])
def test_quest_desc_bruteforce(paged):
    w = small_workload(B=3, len_lo=5, len_hi=29, paged=paged, b=4, d=8, H_kv=2, H_q=4)
    lay, li = make_case(w, seed=3)
    c = oracle_cache(w, lay, li)
    mn, mx = O.quest_desc(c)
    for s in range(w.B):
        for h in range(w.H_kv):
            keys = gather_tokens(c, s, h)
            for j in range(int(c.n_blocks()[s])):
                blk = keys[j * w.b:(j + 1) * w.b]
                assert np.array_equal(mn[s, j, h], blk.min(axis=0))
                assert np.array_equal(mx[s, j, h], blk.max(axis=0))


def test_quest_desc_ignores_tokens_past_len():
    w = small_workload(len_lo=22, len_hi=22)
    lay, li = make_case(w, seed=1)
    c1 = oracle_cache(w, lay, li)
    k2 = li.k.clone()
    k2[5, :, 2:, :] = 100.0  # last page holds tokens 20,21 valid; rows 2,3 are past len
    li2 = W.LayerInputs(li.q, k2, li.v, li.k_new, li.v_new)
    c2 = oracle_cache(w, lay, li2)
    a, b = O.quest_desc(c1), O.quest_desc(c2)
    assert np.array_equal(a[0][:, :6], b[0][:, :6]) and np.array_equal(a[1][:, :6], b[1][:, :6])


def test_gate_desc_against_numpy():
    w = small_workload(B=2, len_lo=9, len_hi=15, d=8, b=4, scorer="gate", dg=6)
    lay, li = make_case(w, seed=5)
    c = oracle_cache(w, lay, li)
    Wk = li.Wk.numpy()
    pooled, kg = O.gate_desc(c, Wk)
    for s in range(w.B):
        for h in range(w.H_kv):
            keys = gather_tokens(c, s, h)
            for j in range(int(c.n_blocks()[s])):
                blk = keys[j * w.b:(j + 1) * w.b]
                want = np.concatenate([blk.max(0), blk.min(0), blk.mean(0)])
                np.testing.assert_allclose(pooled[s, j, h], want, rtol=1e-15, atol=1e-15)
                np.testing.assert_allclose(kg[s, j, h], Wk.astype(np.float64) @ want, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# Quest score
# --------------------------------------------------------------------------

def test_quest_score_is_max_over_box_corners():
    """The per-head Quest score is the maximum of q.x over the key box
    [min, max]: a linear function on a box peaks at a corner (brute force over
    all 2^d corners, d = 4)."""
    w = small_workload(H_q=1, H_kv=1, d=4, b=5, len_lo=20, len_hi=20)
    for seed in range(6):
        lay, li = make_case(w, seed=seed)
        c = oracle_cache(w, lay, li)
        mn, mx = O.quest_desc(c)
        sc = O.quest_scores(c, W.bf16_bits(li.q))
        qv = bf16_to_f64(W.bf16_bits(li.q))[0, 0]
        for j in range(4):
            best = max(sum(qv[ch] * (mx if bit else mn)[0, j, 0, ch] for ch, bit in enumerate(bits))
                       for bits in itertools.product([0, 1], repeat=4))
            assert sc[0, 0, j] == pytest.approx(best, rel=1e-14, abs=1e-14)


def test_quest_score_bounds_group_max_dot():
    w = small_workload(H_q=6, H_kv=2, d=8, b=4, len_lo=37, len_hi=37)
    for seed in range(4):
        lay, li = make_case(w, seed=seed)
        c = oracle_cache(w, lay, li)
        sc = O.quest_scores(c, W.bf16_bits(li.q))
        qv = bf16_to_f64(W.bf16_bits(li.q))[0]
        for h in range(2):
            keys = gather_tokens(c, 0, h)
            for j in range(10):
                blk = keys[j * 4:(j + 1) * 4]
                per_head = [(blk @ qv[h * 3 + i]).max() for i in range(3)]
                assert sc[0, h, j] >= sum(per_head) - 1e-12


def test_quest_score_tight_on_single_token_blocks():
    w = small_workload(H_q=3, H_kv=1, d=8, b=1, len_lo=9, len_hi=9)
    lay, li = make_case(w, seed=2)
    c = oracle_cache(w, lay, li)
    sc = O.quest_scores(c, W.bf16_bits(li.q))
    qv = bf16_to_f64(W.bf16_bits(li.q))[0]
    keys = gather_tokens(c, 0, 0)
    np.testing.assert_allclose(sc[0, 0, :9], keys @ qv.sum(0), rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------
# Selection
# --------------------------------------------------------------------------

def _brute_select(scores, n, L):
    N = len(scores)
    cand = range(N - L)
    best = None
    for sub in itertools.combinations(cand, n - L):
        key = (sum(scores[list(sub)]) if sub else 0.0, [-x for x in sub])
        if best is None or key > best[0]:
            best = (key, sub)
    return sorted(list(best[1]) + list(range(N - L, N)))


@pytest.mark.parametrize("seed", range(12))
def test_select_bruteforce_subsets(seed):
    """Top-n of the non-local blocks = the subset with the largest score sum,
    lowest indices among equal sums; integer scores with many ties."""
    rng = np.random.default_rng(seed)
    N = int(rng.integers(3, 12))
    b = 4
    L = int(rng.integers(0, 3))
    n_budget = int(rng.integers(1, N + 2))
    n_min = int(rng.integers(0, 4))
    scores = rng.integers(-3, 4, size=N).astype(np.float64)
    n = O.num_selected(N, n_budget, L, n_min)
    assert n == min(N, max(min(L, N), n_min, n_budget))
    idx, cnt = O.select(scores.reshape(1, 1, N), np.array([N * b - 1], np.int32), b, n_budget, L, n_min)
    got = list(idx[0, 0, : cnt[0, 0]])
    assert got == _brute_select(scores, n, min(L, N))


def test_select_is_textbook_token_topk():
    """b = 1, one head, no local blocks: the selection is the textbook top-n
    tokens by q.k (numpy lexsort: q.k descending, index ascending)."""
    w = small_workload(H_q=1, H_kv=1, d=8, b=1, len_lo=40, len_hi=40, n_budget=7, n_local=0)
    lay, li = make_case(w, seed=9)
    c = oracle_cache(w, lay, li)
    qv = bf16_to_f64(W.bf16_bits(li.q))[0, 0]
    dots = (gather_tokens(c, 0, 0) @ qv).astype(np.float32)
    order = np.lexsort((np.arange(40), -dots.astype(np.float64)))
    d = O.decode(c, W.bf16_bits(li.q), scale=w.scale, n_budget=7, n_local=0, n_min=0)
    assert list(d.sel_idx[0, 0, : d.sel_cnt[0, 0]]) == sorted(order[:7].tolist())


def test_select_invariants():
    rng = np.random.default_rng(0)
    for _ in range(200):
        N = int(rng.integers(0, 30))
        b = 8
        L = int(rng.integers(0, 5))
        nb, nm = int(rng.integers(0, 40)), int(rng.integers(0, 20))
        sc = rng.normal(size=(1, 1, max(N, 1)))
        ln = N * b - int(rng.integers(0, b)) if N else 0
        idx, cnt = O.select(sc, np.array([ln], np.int32), b, nb, L, nm)
        got = list(idx[0, 0, : cnt[0, 0]])
        n = O.num_selected(N, nb, L, nm)
        assert len(got) == n == (min(N, max(min(L, N), nm, nb)) if N else 0)
        assert got == sorted(set(got))
        assert set(range(max(0, N - L), N)) <= set(got)
        if n >= N:
            assert got == list(range(N))


def test_select_minus_zero_equals_plus_zero():
    sc = np.array([[[-0.0, 0.0, -0.0, 0.0, 1.0]]])
    idx, cnt = O.select(sc, np.array([5], np.int32), 1, 3, 1, 0)
    assert list(idx[0, 0, : cnt[0, 0]]) == [0, 1, 4]


def test_sparsity_budget_rounds_up():
    # keep 5% of 2048 blocks: ceil(102.4) = 103
    assert O.num_selected(2048, 0, 4, 16, 5, 100) == 103
    assert O.num_selected(100, 0, 4, 16, 5, 100) == 16
    assert O.num_selected(3, 64, 2, 16) == 3


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

def _sdpa_dense(c: O.Cache, q_bits, scale):
    """Dense attention through torch's library routine (fp64, CPU)."""
    G = c.H_q // c.H_kv
    outs = []
    for s in range(c.B):
        qs = torch.from_numpy(bf16_to_f64(q_bits)[s])[None, :, None, :]  # [1][H_q][1][d]
        ks = torch.stack([torch.from_numpy(gather_tokens(c, s, h, "k")) for h in range(c.H_kv)])
        vs = torch.stack([torch.from_numpy(gather_tokens(c, s, h, "v")) for h in range(c.H_kv)])
        ks = ks.repeat_interleave(G, 0)[None]
        vs = vs.repeat_interleave(G, 0)[None]
        o = torch.nn.functional.scaled_dot_product_attention(qs, ks, vs, scale=scale)
        outs.append(o[0, :, 0, :].numpy())
    return np.stack(outs)


@pytest.mark.parametrize("paged", [False, True])
def test_select_all_equals_dense_sdpa(paged):
    w = small_workload(B=3, H_q=6, H_kv=2, d=8, b=4, len_lo=7, len_hi=30, paged=paged, n_budget=100)
    lay, li = make_case(w, seed=4)
    c = oracle_cache(w, lay, li)
    q = W.bf16_bits(li.q)
    d = O.decode(c, q, scale=w.scale, n_budget=100, n_local=1, n_min=0)
    np.testing.assert_allclose(d.out, _sdpa_dense(c, q, w.scale), rtol=1e-12, atol=1e-12)


def test_single_token_returns_its_value():
    w = small_workload(B=2, len_lo=1, len_hi=1, H_q=4, H_kv=2)
    lay, li = make_case(w, seed=0)
    c = oracle_cache(w, lay, li)
    d = O.decode(c, W.bf16_bits(li.q), scale=w.scale, n_budget=1, n_local=1, n_min=0)
    for s in range(2):
        for qh in range(4):
            np.testing.assert_array_equal(d.out[s, qh], gather_tokens(c, s, qh // 2, "v")[0])


def test_page_permutation_invariance():
    w = small_workload(B=2, len_lo=30, len_hi=30, paged=True, n_budget=4, n_local=1)
    lay, li = make_case(w, seed=6)
    c = oracle_cache(w, lay, li)
    q = W.bf16_bits(li.q)
    d1 = O.decode(c, q, scale=w.scale, n_budget=4, n_local=1, n_min=0)
    # move every page to a new physical slot (and the table with it)
    perm = np.random.default_rng(1).permutation(lay.num_pages)
    inv = np.argsort(perm)
    k2 = W.bf16_bits(li.k)[inv]
    v2 = W.bf16_bits(li.v)[inv]
    bt2 = np.where(c.block_table >= 0, perm[np.maximum(c.block_table, 0)], -1).astype(np.int32)
    c2 = O.Cache(k2, v2, bt2, c.seq_lens, H_q=w.H_q, max_blocks=c.max_blocks)
    d2 = O.decode(c2, q, scale=w.scale, n_budget=4, n_local=1, n_min=0)
    assert np.array_equal(d1.sel_idx, d2.sel_idx) and np.array_equal(d1.sel_cnt, d2.sel_cnt)
    np.testing.assert_array_equal(d1.out, d2.out)


def test_split_invariance_with_combine():
    w = small_workload(B=2, len_lo=30, len_hi=41, H_q=4, H_kv=2, n_budget=6, n_local=2)
    lay, li = make_case(w, seed=8)
    c = oracle_cache(w, lay, li)
    q = W.bf16_bits(li.q)
    full = O.decode(c, q, scale=w.scale, n_budget=6, n_local=2, n_min=0)
    rng = np.random.default_rng(0)
    for S in (1, 2, 3, 7):
        o_part = np.zeros((w.B, w.H_q, S, w.d))
        l_part = np.zeros((w.B, w.H_q, S))
        for s in range(w.B):
            for h in range(w.H_kv):
                cnt = full.sel_cnt[s, h]
                cuts = np.sort(rng.integers(0, cnt + 1, size=S - 1))
                bounds = [0, *cuts.tolist(), cnt]
                for sp in range(S):
                    sub = full.sel_idx[s, h, bounds[sp]:bounds[sp + 1]]
                    idx = np.zeros((w.B, w.H_kv, max(1, len(sub))), np.int32)
                    cn = np.zeros((w.B, w.H_kv), np.int32)
                    idx[s, h, : len(sub)] = sub
                    cn[s, h] = len(sub)
                    o, l = O.attend(c, q, idx, cn, w.scale)
                    for qh in range(h * w.G, (h + 1) * w.G):
                        o_part[s, qh, sp] = o[s, qh]
                        l_part[s, qh, sp] = l[s, qh]
        out, lse = O.combine(o_part, l_part)
        np.testing.assert_allclose(out, full.out, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse, full.lse, rtol=1e-12, atol=1e-12)


def test_combine_special_cases():
    rng = np.random.default_rng(3)
    o = rng.normal(size=(2, 3, 1, 5))
    l = rng.normal(size=(2, 3, 1))
    out, lse = O.combine(o, l)
    np.testing.assert_array_equal(out, o[:, :, 0])
    np.testing.assert_array_equal(lse, l[:, :, 0])
    o2 = np.concatenate([o, rng.normal(size=(2, 3, 1, 5))], axis=2)
    l2 = np.concatenate([l, np.full((2, 3, 1), -np.inf)], axis=2)
    out2, lse2 = O.combine(o2, l2)
    np.testing.assert_allclose(out2, o[:, :, 0], rtol=1e-15, atol=1e-15)
    out3, lse3 = O.combine(o2, np.full((2, 3, 2), -np.inf))
    assert np.all(out3 == 0) and np.all(lse3 == -np.inf)


def test_empty_sequence():
    w = small_workload(B=2, len_lo=10, len_hi=10)
    lay, li = make_case(w, seed=0)
    c = oracle_cache(w, lay, li)
    c2 = O.Cache(c.k, c.v, None, np.array([0, 10], np.int32), H_q=w.H_q, max_blocks=c.max_blocks)
    d = O.decode(c2, W.bf16_bits(li.q), scale=w.scale, n_budget=2, n_local=1, n_min=0)
    assert np.all(d.sel_cnt[0] == 0) and np.all(d.out[0] == 0) and np.all(d.lse[0] == -np.inf)
    assert np.all(d.sel_cnt[1] == 2)


# --------------------------------------------------------------------------
# Gate and SAS log-gate
# --------------------------------------------------------------------------

def _gate_case(seed=0, **kw):
    base = dict(B=2, H_q=6, H_kv=2, d=8, b=4, len_lo=21, len_hi=33, scorer="gate", dg=8,
                n_budget=4, n_local=2)
    base.update(kw)
    w = small_workload(**base)
    lay, li = make_case(w, seed=seed)
    return w, lay, li, oracle_cache(w, lay, li)


def test_gate_scores_against_library_matmul():
    w, lay, li, c = _gate_case(seed=1)
    q = W.bf16_bits(li.q)
    Wq, Wk = li.Wq.numpy().astype(np.float64), li.Wk.numpy()
    score, logg = O.gate_scores(c, q, li.Wq.numpy(), Wk)
    _, kg = O.gate_desc(c, Wk)
    qf = bf16_to_f64(q)
    for s in range(w.B):
        N = int(c.n_blocks()[s])
        C = N - 1
        for qh in range(w.H_q):
            h = qh // w.G
            u = (kg[s, :C, h] @ (Wq @ qf[s, qh])) / math.sqrt(w.dg)
            lg = torch.log_softmax(torch.from_numpy(u), 0).numpy()
            np.testing.assert_allclose(logg[s, qh, :C], lg, rtol=1e-12, atol=1e-12)
            assert logg[s, qh, N - 1] == 0.0  # current block B0: unit gate
            assert np.exp(logg[s, qh, :C]).sum() == pytest.approx(1.0, abs=1e-12)
        for h in range(w.H_kv):
            g = np.exp(logg[s, h * w.G:(h + 1) * w.G, :C]).sum(0)
            np.testing.assert_allclose(score[s, h, :C], g, rtol=1e-12, atol=1e-14)
            assert score[s, h, :C].sum() == pytest.approx(w.G, abs=1e-12)


def test_gate_equal_blocks_give_uniform_log_gate():
    """Identical blocks -> identical pooled keys -> equal u -> log g = -log C."""
    w, lay, li, c = _gate_case(seed=2, B=1, len_lo=24, len_hi=24, paged=False)
    k = li.k.clone()
    k[:] = k[0:1]
    li2 = W.LayerInputs(li.q, k, li.v, li.k_new, li.v_new, li.Wq, li.Wk)
    c2 = oracle_cache(w, lay, li2)
    _, logg = O.gate_scores(c2, W.bf16_bits(li.q), li.Wq.numpy(), li.Wk.numpy())
    C = 24 // 4 - 1
    np.testing.assert_allclose(logg[0, :, :C], -math.log(C), rtol=1e-12)


def test_gate_single_historical_block_is_unbiased():
    """C = 1 -> g = 1 -> log g = 0: gated attention equals plain attention."""
    w, lay, li, c = _gate_case(seed=3, B=1, len_lo=7, len_hi=7)
    q = W.bf16_bits(li.q)
    dg = O.decode(c, q, scale=w.scale, n_budget=4, n_local=2, n_min=0, scorer="gate",
                  Wq=li.Wq.numpy(), Wk=li.Wk.numpy())
    assert np.all(dg.logg[0, :, :2] == 0.0)
    dq = O.decode(c, q, scale=w.scale, n_budget=4, n_local=2, n_min=0)
    np.testing.assert_array_equal(dg.out, dq.out)


def test_log_gate_inside_softmax_equals_gate_weighted_form():
    """softmax(l + log g) V == sum_t g_j(t) e^{l_t} v_t / sum_t g_j(t) e^{l_t}."""
    w, lay, li, c = _gate_case(seed=4)
    q = W.bf16_bits(li.q)
    d = O.decode(c, q, scale=w.scale, n_budget=4, n_local=2, n_min=0, scorer="gate",
                 Wq=li.Wq.numpy(), Wk=li.Wk.numpy())
    qf = bf16_to_f64(q)
    for s in range(w.B):
        L = int(c.seq_lens[s])
        for qh in range(w.H_q):
            h = qh // w.G
            keys, vals = gather_tokens(c, s, h, "k"), gather_tokens(c, s, h, "v")
            sel = d.sel_idx[s, h, : d.sel_cnt[s, h]]
            toks = [t for j in sel for t in range(j * w.b, min((j + 1) * w.b, L))]
            l = keys[toks] @ qf[s, qh] * w.scale
            gate = np.exp(np.array([d.logg[s, qh, t // w.b] for t in toks]))
            wts = gate * np.exp(l - l.max())
            np.testing.assert_allclose(d.out[s, qh], wts @ vals[toks] / wts.sum(), rtol=1e-12, atol=1e-13)
