"""Pins of the SAS gate variants in the CPU oracle (oracle/sas_variants.py).

Each pin is fixed by the page's formulas or by mathematics: the inner softmax
variant is the method's own form (and must equal the main oracle's gated
decode), unit gates make every variant plain attention, the outer form is a
gate-weighted sum under ungated softmax weights (written out here with numpy
vectors), the sigmoid log-gate is numpy's -logaddexp(0, -u) without overflow, and a
one-head group ranks blocks by the gate itself (a textbook top-k).
"""
from __future__ import annotations

import math

import numpy as np
import pytest

import oracle as O
from oracle import sas_variants as V
from block_sparse_gqa_min_b200 import workloads as W
from tests.helpers import bf16_to_f64, gather_tokens, make_case, oracle_cache, small_workload


def _case(seed=0, **kw):
    base = dict(B=2, H_q=6, H_kv=2, d=8, b=4, len_lo=21, len_hi=33, scorer="gate", dg=8, n_budget=4, n_local=2)
    base.update(kw)
    w = small_workload(**base)
    lay, li = make_case(w, seed=seed)
    return w, li, oracle_cache(w, lay, li)


def _run(w, li, c, **kw):
    return V.decode_variant(c, W.bf16_bits(li.q), li.Wq.numpy(), li.Wk.numpy(), scale=w.scale,
                            n_budget=w.n_budget, n_local=w.n_local, n_min=0, **kw)


@pytest.mark.parametrize("seed", range(3))
def test_inner_softmax_is_the_main_gated_decode(seed):
    w, li, c = _case(seed)
    ref = O.decode(c, W.bf16_bits(li.q), scale=w.scale, n_budget=w.n_budget, n_local=w.n_local, n_min=0,
                   scorer="gate", Wq=li.Wq.numpy(), Wk=li.Wk.numpy())
    got = _run(w, li, c, activation="softmax", position="inner")
    np.testing.assert_array_equal(got.sel_idx, ref.sel_idx)
    np.testing.assert_array_equal(got.sel_cnt, ref.sel_cnt)
    fin = np.isfinite(ref.logg)
    np.testing.assert_allclose(got.logg[fin], ref.logg[fin], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got.out, ref.out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got.lse, ref.lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("position", V.POSITIONS)
def test_unit_gates_give_plain_attention(position):
    """Wq = 0 makes every gate logit 0; raw injection then gives g = 1 on every
    block, and both positions reduce to softmax(qK^T)V over the selection."""
    w, li, c = _case(4)
    Wq0 = np.zeros_like(li.Wq.numpy())
    q = W.bf16_bits(li.q)
    got = V.decode_variant(c, q, Wq0, li.Wk.numpy(), scale=w.scale, n_budget=w.n_budget, n_local=w.n_local,
                           n_min=0, activation="raw", position=position)
    assert np.all(got.logg[np.isfinite(got.logg)] == 0.0)
    o, l = O.attend(c, q, got.sel_idx, got.sel_cnt, w.scale)
    np.testing.assert_allclose(got.out, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got.lse, l, rtol=0, atol=1e-12)


@pytest.mark.parametrize("activation", V.ACTIVATIONS)
def test_outer_is_gate_weighted_values_under_ungated_softmax(activation):
    w, li, c = _case(5)
    d = _run(w, li, c, activation=activation, position="outer")
    qf = bf16_to_f64(W.bf16_bits(li.q))
    for s in range(w.B):
        L = int(c.seq_lens[s])
        for qh in range(w.H_q):
            h = qh // w.G
            keys, vals = gather_tokens(c, s, h, "k"), gather_tokens(c, s, h, "v")
            sel = d.sel_idx[s, h, : d.sel_cnt[s, h]]
            toks = np.array([t for j in sel for t in range(j * w.b, min((j + 1) * w.b, L))])
            logits = keys[toks] @ qf[s, qh] * w.scale
            p = np.exp(logits - logits.max())
            p /= p.sum()
            g = np.exp(d.logg[s, qh, toks // w.b])
            np.testing.assert_allclose(d.out[s, qh], (p * g) @ vals[toks], rtol=1e-12, atol=1e-13)
            m = logits.max()
            assert d.lse[s, qh] == pytest.approx(m + math.log(np.exp(logits - m).sum()), rel=1e-12)


def test_sigmoid_log_gate():
    u = np.linspace(-30.0, 30.0, 121)
    # log(1 / (1 + e^-u)) = -log(e^0 + e^-u): numpy's logaddexp
    np.testing.assert_allclose(V.log_gates(u, "sigmoid"), -np.logaddexp(0.0, -u), rtol=1e-13, atol=0)
    big = V.log_gates(np.array([-800.0, 800.0]), "sigmoid")
    assert big[0] == -800.0 and big[1] == 0.0           # no overflow either side
    assert np.all(V.log_gates(u, "sigmoid") < 0.0)
    sm = V.log_gates(u, "softmax")
    assert np.exp(sm).sum() == pytest.approx(1.0, abs=1e-12)
    np.testing.assert_array_equal(V.log_gates(u, "raw"), u)


@pytest.mark.parametrize("activation", V.ACTIVATIONS)
def test_one_head_group_ranks_by_its_gate(activation):
    """G = 1: the group score is the head's own gate, so the historical blocks
    chosen are the top (n - L) by fp32 gate value, lower index first on ties."""
    w, li, c = _case(6, H_q=2, H_kv=2, len_lo=40, len_hi=40, n_budget=5, n_local=1)
    d = _run(w, li, c, activation=activation, position="inner")
    N = 10
    n = O.num_selected(N, 5, 1, 0)
    for s in range(w.B):
        for h in range(w.H_kv):
            g = np.exp(d.logg[s, h, : N - 1]).astype(np.float32)
            order = np.lexsort((np.arange(N - 1), -g.astype(np.float64)))
            expect = sorted(order[: n - 1].tolist() + [N - 1])
            assert list(d.sel_idx[s, h, : d.sel_cnt[s, h]]) == expect
