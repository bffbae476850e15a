"""Pins of the multi-token oracle (oracle/multi_query.py): several query tokens
of a sequence sharing one selection, each attending causally; the dense
rectification pass as the select-all case.

Pins: one token is the main decode; the shared score is the main score of a
group whose heads are the (token, head) pairs (the score is a sum over heads);
each token's output is softmax attention over the selected tokens up to its own
position (written out with numpy); the dense pass is torch's causal
scaled_dot_product_attention over the whole cache.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from oracle import multi_query as MQ
from block_sparse_gqa_min_b200 import workloads as W
from tests.helpers import bf16_to_f64, gather_tokens, make_case, oracle_cache, small_workload


def _case(seed, M, **kw):
    base = dict(B=2, H_q=6, H_kv=2, d=8, b=4, len_lo=19, len_hi=37, n_budget=4, n_local=2)
    base.update(kw)
    w = small_workload(**base)
    lay, li = make_case(w, seed=seed)
    c = oracle_cache(w, lay, li)
    g = torch.Generator().manual_seed(seed + 101)
    q = W.bf16_bits(torch.randn((w.B, M, w.H_q, w.d), generator=g).to(torch.bfloat16))
    return w, c, q


def test_one_token_is_the_main_decode():
    w, c, q = _case(0, 1)
    score, si, sc, out, lse = MQ.decode_multi(c, q, scale=w.scale, n_budget=4, n_local=2, n_min=0)
    ref = O.decode(c, np.ascontiguousarray(q[:, 0]), scale=w.scale, n_budget=4, n_local=2, n_min=0)
    np.testing.assert_array_equal(si, ref.sel_idx)
    np.testing.assert_array_equal(sc, ref.sel_cnt)
    np.testing.assert_array_equal(out[:, 0], ref.out)
    np.testing.assert_array_equal(lse[:, 0], ref.lse)


@pytest.mark.parametrize("M", [2, 3])
def test_shared_score_is_the_score_of_a_wider_group(M):
    """The M tokens of a group act as M*G heads of one group."""
    w, c, q = _case(1, M)
    score, *_ = MQ.decode_multi(c, q, scale=w.scale, n_budget=4, n_local=2, n_min=0)
    G = w.G
    q2 = np.zeros((w.B, w.H_kv * M * G, w.d), dtype=np.uint16)
    for g in range(w.H_kv):
        for i in range(M):
            for hh in range(G):
                q2[:, g * M * G + i * G + hh] = q[:, i, g * G + hh]
    wide = O.Cache(c.k, c.v, c.block_table, c.seq_lens, H_q=w.H_q * M, max_blocks=c.max_blocks)
    ref = O.quest_scores(wide, q2)
    N = c.n_blocks()
    for s in range(w.B):
        np.testing.assert_allclose(score[s, :, : N[s]], ref[s, :, : N[s]], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed", range(3))
def test_each_token_attends_causally_over_the_shared_selection(seed):
    M = 3
    w, c, q = _case(seed + 2, M)
    _, si, sc, out, lse = MQ.decode_multi(c, q, scale=w.scale, n_budget=4, n_local=2, n_min=0)
    qf = bf16_to_f64(q)
    for s in range(w.B):
        L = int(c.seq_lens[s])
        for i in range(M):
            horizon = L - M + i + 1
            for qh in range(w.H_q):
                h = qh // w.G
                keys, vals = gather_tokens(c, s, h, "k"), gather_tokens(c, s, h, "v")
                sel = si[s, h, : sc[s, h]]
                toks = np.array([t for j in sel for t in range(j * w.b, (j + 1) * w.b) if t < horizon])
                lg = keys[toks] @ qf[s, i, qh] * w.scale
                p = np.exp(lg - lg.max())
                np.testing.assert_allclose(out[s, i, qh], (p / p.sum()) @ vals[toks], rtol=1e-12, atol=1e-13)
                assert lse[s, i, qh] == pytest.approx(lg.max() + np.log(p.sum()), rel=1e-12)


def test_dense_rectification_pass_is_causal_sdpa():
    """Every block selected: token i of the last f = 4 attends to all positions
    up to its own, as torch's scaled_dot_product_attention with that mask."""
    f = 4
    w, c, q = _case(7, f, B=1, len_lo=30, len_hi=30)
    _, si, sc, out, _ = MQ.decode_multi(c, q, scale=w.scale, n_budget=0, n_local=0, n_min=0, dense=True)
    assert np.all(sc == c.n_blocks()[0])
    L = 30
    mask = torch.tensor([[t <= L - f + i for t in range(L)] for i in range(f)])
    qf = torch.from_numpy(bf16_to_f64(q))[0]                                  # [f][H_q][d]
    for qh in range(w.H_q):
        h = qh // w.G
        k = torch.from_numpy(gather_tokens(c, 0, h, "k"))
        v = torch.from_numpy(gather_tokens(c, 0, h, "v"))
        ref = torch.nn.functional.scaled_dot_product_attention(qf[:, qh][None], k[None], v[None], attn_mask=mask[None],
                                                               scale=w.scale)[0]
        np.testing.assert_allclose(out[0, :, qh], ref.numpy(), rtol=1e-12, atol=1e-12)
