"""GPU parity of the fused one-launch decode step (sba_decode_step) against the
CPU oracle run on the cache as it stands after the step's append."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_gqa_min_b200 import sba
from block_sparse_gqa_min_b200 import workloads as W
from tests.helpers import (ATOL_OUT, check_selection, fill_descriptors, gpu_cache, oracle_cache, oracle_decode,
                           params_of, small_workload)
from tests.test_parity_gpu import check_descriptors

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def run_fused(w: W.Workload, seed=0, n_app=0, layout=None, layer_inputs=None, device="cpu", out_dtype=torch.float32,
              pos_back=0):
    lay = layout or W.make_layout(w, seed, device=device)
    li = layer_inputs or W.make_layer(w, lay, seed, 0, device=device)
    c = gpu_cache(w, lay, li)
    fill_descriptors(c, w, li)
    p = params_of(w)
    dev = torch.device("cuda")
    A = None
    if w.scorer == "gate":
        A = torch.empty((w.d, 3 * w.d), dtype=torch.float32, device=dev)
        sba.sba_fold_gate(li.Wq.to(dev), li.Wk.to(dev), A)
    N_max = (c.max_len + w.b - 1) // w.b
    n_max = max(1, sba.sba_num_selected(N_max, p))
    sel_idx = torch.full((w.B, w.H_kv, n_max), -1, dtype=torch.int32, device=dev)
    sel_cnt = torch.zeros((w.B, w.H_kv), dtype=torch.int32, device=dev)
    gbias = torch.zeros((w.B, w.H_q, n_max), dtype=torch.float32, device=dev) if w.scorer == "gate" else None
    out = torch.empty((w.B, w.H_q, w.d), dtype=out_dtype, device=dev)
    lse = torch.empty((w.B, w.H_q), dtype=torch.float32, device=dev)
    kw = {}
    if n_app:
        g = torch.Generator().manual_seed(seed + 77)
        kw = dict(k_new=torch.randn((w.B, n_app, w.H_kv, w.d), generator=g).to(torch.bfloat16).to(dev),
                  v_new=torch.randn((w.B, n_app, w.H_kv, w.d), generator=g).to(torch.bfloat16).to(dev),
                  pos_start=(c.seq_lens - n_app - pos_back).clamp(min=0).to(torch.int32))
    sba.sba_decode_step(c, li.q.to(dev), p, w.scale, out, lse, gate_A=A, sel_idx=sel_idx, sel_cnt=sel_cnt,
                        gate_bias=gbias, **kw)
    torch.cuda.synchronize()
    assert int(c.status.item()) == 0
    # the oracle sees the cache after the append
    li2 = W.LayerInputs(li.q, c.k.cpu(), c.v.cpu(), li.k_new, li.v_new, li.Wq, li.Wk)
    oc = oracle_cache(w, lay, li2)
    ref = oracle_decode(w, oc, li2, n_max=n_max)
    si, sc = sel_idx.cpu().numpy(), sel_cnt.cpu().numpy()
    events = check_selection(ref, si, sc, oc, w)
    expect = ref
    if events:  # near-ties: the oracle's step re-run on the GPU's selection
        expect = oracle_decode(w, oc, li2, n_max=n_max, sel=(si, sc))
    got = out.float().cpu().numpy()
    tol = ATOL_OUT if out_dtype == torch.float32 else ATOL_OUT + np.abs(expect.out).max() / 256
    err = float(np.abs(got - expect.out).max())
    assert err <= tol, err
    lg = lse.cpu().numpy()
    fin = np.isfinite(expect.lse)
    assert np.array_equal(np.isfinite(lg), fin)
    assert np.abs(lg[fin] - expect.lse[fin]).max(initial=0) <= 1e-3
    if w.scorer == "gate":
        gb = gbias.cpu().numpy()
        for s in range(w.B):
            for qh in range(w.H_q):
                n = sc[s, qh // w.G]
                np.testing.assert_allclose(gb[s, qh, :n], expect.logg[s, qh, si[s, qh // w.G, :n]], rtol=0,
                                           atol=5e-5)
    if n_app:
        check_descriptors(w, lay, li2, c, oc)
    return dict(events=events, err=err, c=c, sel_idx=si, sel_cnt=sc, ref=ref)


FUSED_CASES = [
    dict(H_q=8, H_kv=2, b=64, len_lo=4096, len_hi=4096, n_budget=16, n_local=2, hot_blocks=4),   # tiny-like
    dict(H_q=32, H_kv=8, b=64, len_lo=20000, len_hi=20000, n_budget=64, n_local=2, n_min=16,
         channel_scale_sigma=0.5),
    dict(H_q=28, H_kv=4, b=128, len_lo=30000, len_hi=30000, n_local=4, n_min=16, keep_num=5, keep_den=100),
    dict(H_q=32, H_kv=8, b=64, len_lo=3000, len_hi=9000, B=3, n_budget=32, n_local=2, n_min=16, paged=True),
    dict(H_q=16, H_kv=1, b=64, len_lo=77, len_hi=77, n_budget=4, n_local=1),         # G 16, 2 blocks
    dict(H_q=4, H_kv=4, b=64, len_lo=1, len_hi=1, n_budget=4, n_local=1),            # one token
    dict(H_q=8, H_kv=8, b=128, len_lo=1000, len_hi=1000, n_budget=100, n_local=2),  # select all
    dict(H_q=6, H_kv=3, b=64, len_lo=64, len_hi=5000, B=5, n_budget=3, n_local=1, paged=True),
    # contiguous pages, lengths that differ: slices are fixed shares of max_blocks, so the CTAs
    # past a short sequence's end drain their early descriptor loads unread
    dict(H_q=8, H_kv=2, b=64, len_lo=100, len_hi=6000, B=4, n_budget=8, n_local=2),
]


@pytest.mark.parametrize("case", range(len(FUSED_CASES)))
@pytest.mark.parametrize("n_app", [0, 1])
def test_fused_quest(case, n_app):
    w = small_workload(d=128, **FUSED_CASES[case])
    run_fused(w, seed=case, n_app=n_app)


def test_fused_rectification_window():
    """A 32-token window spanning two b=128 blocks, both local (L = 4)."""
    w = small_workload(d=128, H_q=28, H_kv=4, b=128, len_lo=30000, len_hi=30000, n_local=4, n_min=16,
                       keep_num=5, keep_den=100)
    run_fused(w, seed=5, n_app=32)


def test_fused_refreshes_scored_block_first():
    """No local blocks: the appended block is itself ranked, so it is
    refreshed before scoring (extra cluster barrier)."""
    w = small_workload(d=128, H_q=8, H_kv=2, b=64, len_lo=3000, len_hi=3000, n_budget=6, n_local=0)
    run_fused(w, seed=2, n_app=1)
    run_fused(w, seed=3, n_app=40)


def test_fused_refresh_inside_fill_loop():
    """Tokens overwritten inside an early local block (12 local blocks, two CTAs per
    cluster): the touched block is followed by more fills than the ring holds, so its
    descriptor is rebuilt inside the producer's fill loop, not after it."""
    w = small_workload(d=128, H_q=16, H_kv=8, b=64, len_lo=3000, len_hi=3000, B=8, n_budget=24, n_local=12)
    run_fused(w, seed=4, n_app=40, pos_back=64 * 10)


FUSED_GATE_CASES = [
    dict(H_q=40, H_kv=8, b=64, len_lo=30000, len_hi=30000, n_budget=32, n_local=2, n_min=16),
    dict(H_q=10, H_kv=2, b=64, len_lo=3000, len_hi=7000, B=2, n_budget=6, n_local=2, paged=True),
    dict(H_q=5, H_kv=1, b=64, len_lo=65, len_hi=65, n_budget=4, n_local=2),          # C = 1 historical
    dict(H_q=8, H_kv=4, b=128, len_lo=200, len_hi=5000, B=3, n_budget=5, n_local=0, paged=True),
    dict(H_q=10, H_kv=2, b=64, len_lo=300, len_hi=6000, B=3, n_budget=6, n_local=2),  # contiguous, lengths differ
    dict(H_q=32, H_kv=2, b=128, len_lo=9000, len_hi=9000, n_budget=8, n_local=2),      # G 16: two 8-head tiles
    dict(H_q=32, H_kv=2, b=64, len_lo=2000, len_hi=9000, B=2, n_budget=10, n_local=1, paged=True),  # G 16, paged
]


@pytest.mark.parametrize("case", range(len(FUSED_GATE_CASES)))
@pytest.mark.parametrize("n_app", [0, 1])
def test_fused_gate(case, n_app):
    w = small_workload(d=128, scorer="gate", dg=128, **FUSED_GATE_CASES[case])
    run_fused(w, seed=case, n_app=n_app)


def test_fused_gate_window_touching_historical_block():
    """A window reaching back into block N-2 (historical for the gate): refreshed before scoring."""
    w = small_workload(d=128, scorer="gate", dg=128, H_q=10, H_kv=2, b=64, len_lo=3000, len_hi=3000,
                       n_budget=6, n_local=2)
    run_fused(w, seed=1, n_app=90)


def test_fused_bf16_output():
    w = small_workload(d=128, H_q=32, H_kv=8, b=64, len_lo=20000, len_hi=20000, n_budget=64, n_local=2)
    run_fused(w, seed=0, n_app=1, out_dtype=torch.bfloat16)


def test_fused_equals_separate_calls_on_exact_ties():
    """Duplicated pages give exactly equal scores: lower index must win in the
    fused path too."""
    w = small_workload(d=128, H_q=8, H_kv=2, b=64, len_lo=64 * 40, len_hi=64 * 40, n_budget=5, n_local=1)
    lay = W.make_layout(w, 0)
    li = W.make_layer(w, lay, 0, 0)
    for p in (3, 7, 19, 25, 33):
        li.k[p] = li.k[2]
    r = run_fused(w, 0, layout=lay, layer_inputs=li)
    assert r["events"] == 0


# SAS gate variants ("SAS ...", Method: the gate inside the softmax or on the values; softmax,
# sigmoid and unnormalised activations), and the gate used for selection only.
GATE_VARIANTS = [(pos, act) for pos in ("inner", "outer") for act in ("softmax", "sigmoid", "raw")]


@pytest.mark.parametrize("pos,act", GATE_VARIANTS)
@pytest.mark.parametrize("case", [0, 1, 2])
def test_fused_gate_variants(pos, act, case):
    shapes = [dict(H_q=40, H_kv=8, b=64, len_lo=30000, len_hi=30000, n_budget=32, n_local=2, n_min=16),
              dict(H_q=10, H_kv=2, b=64, len_lo=3000, len_hi=7000, B=2, n_budget=6, n_local=2, paged=True),
              dict(H_q=32, H_kv=2, b=128, len_lo=5000, len_hi=9000, B=2, n_budget=8, n_local=1)]
    w = small_workload(d=128, scorer="gate", dg=128, gate_position=pos, gate_act=act, **shapes[case])
    run_fused(w, seed=11 + case, n_app=1)


@pytest.mark.parametrize("act", ["softmax", "sigmoid"])
def test_fused_gate_selects_without_log_gate(act):
    """log_gate off: the gate ranks the blocks, the attention over them is plain."""
    w = small_workload(d=128, scorer="gate", dg=128, gate_position="off", gate_act=act, H_q=40, H_kv=8, b=64,
                       len_lo=30000, len_hi=30000, n_budget=32, n_local=2, n_min=16)
    r = run_fused(w, seed=21, n_app=1)
    # the same selection with the log-gate inside the softmax gives a different output
    w2 = w.with_(gate_position="inner")
    r2 = run_fused(w2, seed=21, n_app=1)
    assert np.array_equal(r["sel_idx"], r2["sel_idx"])
