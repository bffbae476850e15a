"""GPU parity of the multi-token calls against the CPU oracle (oracle.multi_query):
several query tokens sharing one selection (sba_score_select_multi +
sba_sparse_decode_multi + sba_combine) and the dense causal rectification pass
(sba_rectify), which also writes the tokens' K/V and refreshes the touched
blocks' descriptors.

Selections must match bit-exactly (near-ties of the oracle's own scores within
1e-5 relative are resolved by re-running the oracle on the GPU's selection);
outputs within 2e-3 max-abs, LSE within 1e-3; the cache rows and the Quest
descriptors exactly."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_gqa_min_b200 import sba
from block_sparse_gqa_min_b200 import workloads as W
from oracle import multi_query as MQ
from tests.helpers import (ATOL_OUT, check_selection, fill_descriptors, gpu_cache, oracle_cache, params_of,
                           small_workload)
from tests.test_parity_gpu import check_descriptors

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def multi_q(w: W.Workload, M: int, seed: int) -> torch.Tensor:
    """Seeded query tokens [B][M][H_q][d] (bf16, N(0,1))."""
    g = torch.Generator().manual_seed(seed * 131 + M)
    return torch.randn((w.B, M, w.H_q, w.d), generator=g).to(torch.bfloat16)


def splits_for(c, M, n_blocks, num_sms=148):
    rg = sba.sba_multi_row_groups(c, M)
    return max(1, min(n_blocks, num_sms // max(1, c.B * c.H_kv * rg)))


def check_out(out, lse, exp_out, exp_lse):
    err = float(np.abs(out - exp_out).max())
    assert err <= ATOL_OUT, err
    fin = np.isfinite(exp_lse)
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.abs(lse[fin] - exp_lse[fin]).max(initial=0) <= 1e-3
    return err


def run_multi(w: W.Workload, M: int, seed=0, num_splits=None):
    lay = W.make_layout(w, seed)
    li = W.make_layer(w, lay, seed, 0)
    c = gpu_cache(w, lay, li)
    fill_descriptors(c, w, li)
    p = params_of(w)
    dev = torch.device("cuda")
    q = multi_q(w, M, seed)
    N_max = (c.max_len + w.b - 1) // w.b
    n_max = max(1, sba.sba_num_selected(N_max, p))
    sel_idx = torch.full((w.B, w.H_kv, n_max), -1, dtype=torch.int32, device=dev)
    sel_cnt = torch.zeros((w.B, w.H_kv), dtype=torch.int32, device=dev)
    ws = torch.zeros((sba.sba_workspace_size(c, p) + 15) // 16 * 16, dtype=torch.uint8, device=dev)
    S = num_splits or splits_for(c, M, n_max)
    o_part = torch.empty((w.B, M, w.H_q, S, w.d), dtype=torch.float32, device=dev)
    lse_part = torch.empty((w.B, M, w.H_q, S), dtype=torch.float32, device=dev)
    out = torch.empty((w.B, M, w.H_q, w.d), dtype=torch.float32, device=dev)
    lse = torch.empty((w.B, M, w.H_q), dtype=torch.float32, device=dev)
    qd = q.to(dev)
    sba.sba_score_select_multi(c, qd, p, sel_idx, sel_cnt, ws)
    sba.sba_sparse_decode_multi(c, qd, sel_idx, sel_cnt, w.scale, o_part, lse_part)
    sba.sba_combine(o_part, lse_part, out.view(w.B, M * w.H_q, w.d), lse.view(w.B, M * w.H_q))
    torch.cuda.synchronize()
    assert int(c.status.item()) == 0
    oc = oracle_cache(w, lay, li)
    kw = dict(scale=w.scale, n_budget=w.n_budget, n_local=w.n_local, n_min=w.n_min, keep_num=w.keep_num,
              keep_den=w.keep_den, n_max=n_max)
    qb = W.bf16_bits(q)
    score, ri, rc, ro, rl = MQ.decode_multi(oc, qb, **kw)
    si, sc = sel_idx.cpu().numpy(), sel_cnt.cpu().numpy()
    events = check_selection(O.Decoded(score, ri, rc, None, ro, rl), si, sc, oc, w)
    if events:  # near-ties: the oracle re-run on the GPU's selection
        _, _, _, ro, rl = MQ.decode_multi(oc, qb, sel=(si, sc), **kw)
    err = check_out(out.cpu().numpy(), lse.cpu().numpy(), ro, rl)
    return dict(events=events, err=err)


MULTI_CASES = [
    dict(H_q=32, H_kv=8, b=64, len_lo=20000, len_hi=20000, n_budget=64, n_local=2, n_min=16,
         channel_scale_sigma=0.5),                                                          # G 4
    dict(H_q=28, H_kv=4, b=128, len_lo=30000, len_hi=30000, n_local=4, n_min=16, keep_num=5, keep_den=100),  # G 7
    dict(H_q=8, H_kv=2, b=64, len_lo=300, len_hi=6000, B=3, n_budget=8, n_local=2, paged=True),  # ragged, paged
]


@pytest.mark.parametrize("M", [1, 4, 32])
@pytest.mark.parametrize("case", range(len(MULTI_CASES)))
def test_multi_query_sparse(case, M):
    w = small_workload(d=128, **MULTI_CASES[case])
    run_multi(w, M, seed=case)


def test_multi_query_split_counts_agree():
    w = small_workload(d=128, **MULTI_CASES[2])
    for S in (1, 3, 7):
        run_multi(w, 5, seed=9, num_splits=S)


def test_multi_query_rows_beyond_one_cta():
    """G 16 x 20 tokens = 320 query rows: three row groups of up to 128."""
    w = small_workload(d=128, H_q=16, H_kv=1, b=64, len_lo=2000, len_hi=2000, n_budget=8, n_local=2)
    run_multi(w, 20, seed=3)


@pytest.mark.parametrize("M,shape", [
    (128, dict(H_q=8, H_kv=2, b=64, len_lo=3000, len_hi=3000, n_budget=16, n_local=2)),     # 512 rows, 4 row groups
    (1024, dict(H_q=2, H_kv=2, b=128, len_lo=2100, len_hi=4000, B=2, n_budget=8, n_local=2,
                paged=True)),                                                                # M at its limit, G 1
])
def test_multi_query_many_rows(M, shape):
    w = small_workload(d=128, **shape)
    run_multi(w, M, seed=M)


def test_multi_query_short_sequences():
    """Sequences shorter than a block and exactly M tokens long (every token a query)."""
    w = small_workload(d=128, H_q=8, H_kv=2, b=64, len_lo=4, len_hi=70, B=4, n_budget=2, n_local=1, paged=True)
    run_multi(w, 4, seed=1)


# ---------------------------------------------------------------------------
# rectification: dense causal attention of the last f tokens, with their KV write
# ---------------------------------------------------------------------------

def run_rectify(w: W.Workload, f: int, seed=0, num_splits=None):
    lay = W.make_layout(w, seed)
    li = W.make_layer(w, lay, seed, 0)
    c = gpu_cache(w, lay, li)
    fill_descriptors(c, w, li)  # descriptors of the cache BEFORE the window is rewritten
    dev = torch.device("cuda")
    q = multi_q(w, f, seed)
    g = torch.Generator().manual_seed(seed + 991)
    kn = torch.randn((w.B, f, w.H_kv, w.d), generator=g).to(torch.bfloat16)
    vn = torch.randn((w.B, f, w.H_kv, w.d), generator=g).to(torch.bfloat16)
    N_max = (c.max_len + w.b - 1) // w.b
    S = num_splits or splits_for(c, f, N_max)
    o_part = torch.empty((w.B, f, w.H_q, S, w.d), dtype=torch.float32, device=dev)
    lse_part = torch.empty((w.B, f, w.H_q, S), dtype=torch.float32, device=dev)
    out = torch.empty((w.B, f, w.H_q, w.d), dtype=torch.float32, device=dev)
    lse = torch.empty((w.B, f, w.H_q), dtype=torch.float32, device=dev)
    sba.sba_rectify(c, q.to(dev), kn.to(dev), vn.to(dev), w.scale, o_part, lse_part)
    sba.sba_combine(o_part, lse_part, out.view(w.B, f * w.H_q, w.d), lse.view(w.B, f * w.H_q))
    torch.cuda.synchronize()
    assert int(c.status.item()) == 0
    # the expected cache: the window's rows written through the block table
    k2, v2 = li.k.clone(), li.v.clone()
    for s in range(w.B):
        L = int(lay.seq_lens[s])
        for i in range(f):
            t = L - f + i
            page = int(lay.block_table[s, t // w.b]) if lay.block_table is not None else s * lay.max_blocks + t // w.b
            k2[page, :, t % w.b] = kn[s, i]
            v2[page, :, t % w.b] = vn[s, i]
    assert torch.equal(c.k.cpu(), k2) and torch.equal(c.v.cpu(), v2), "cache rows differ"
    li2 = W.LayerInputs(li.q, k2, v2, kn, vn)
    oc = oracle_cache(w, lay, li2)
    check_descriptors(w, lay, li2, c, oc)  # every block, the refreshed ones included, exactly
    _, _, _, ro, rl = MQ.decode_multi(oc, W.bf16_bits(q), scale=w.scale, n_budget=0, n_local=0, n_min=0,
                                      dense=True, n_max=N_max)
    return check_out(out.cpu().numpy(), lse.cpu().numpy(), ro, rl)


RECT_CASES = [
    (dict(H_q=28, H_kv=4, b=128, len_lo=12000, len_hi=12000, n_local=4), 32),        # R1 shape, f 32
    (dict(H_q=32, H_kv=8, b=64, len_lo=6000, len_hi=6000, n_local=2), 16),          # f 16
    (dict(H_q=8, H_kv=2, b=64, len_lo=300, len_hi=5000, B=3, n_local=2, paged=True), 128),  # 3 blocks touched
    (dict(H_q=8, H_kv=2, b=128, len_lo=1000, len_hi=4000, B=2, n_local=2), 64),     # window inside a block
    (dict(H_q=4, H_kv=1, b=64, len_lo=64, len_hi=64, n_local=1), 64),               # every token new
    (dict(H_q=8, H_kv=2, b=128, len_lo=1000, len_hi=1000, n_local=2), 128),         # 128 tokens over 2 blocks
    (dict(H_q=32, H_kv=2, b=64, len_lo=3000, len_hi=3000, n_local=2), 16),          # 256 rows: 2 row groups
    (dict(H_q=16, H_kv=1, b=128, len_lo=4000, len_hi=9000, B=2, n_local=2, paged=True), 32),  # G 16: 4 row groups
    (dict(H_q=7, H_kv=1, b=64, len_lo=129, len_hi=129, n_local=1), 128),            # f = 128 over 3 blocks, 896 rows
]


@pytest.mark.parametrize("case", range(len(RECT_CASES)))
def test_rectify(case):
    shape, f = RECT_CASES[case]
    w = small_workload(d=128, **shape)
    run_rectify(w, f, seed=case)


def test_rectify_split_counts_agree():
    shape, f = RECT_CASES[2]
    w = small_workload(d=128, **shape)
    for S in (1, 2, 9):
        run_rectify(w, f, seed=7, num_splits=S)
