"""The allocation-free scoring entry point (sba_score_select_static).

Callers that cannot allocate device memory when they issue a step -- an
engine recording its step into a CUDA graph, which forbids cudaMalloc during
capture, or a framework plugin whose enqueue callback must not allocate --
call sba_score_select_static, which uses the library's static per-device
scratch instead of a caller workspace.  Its results must equal those of
sba_score_select with a caller workspace, call after call (the static scratch
keeps the previous call's contents, so two calls in a row are checked)."""
from __future__ import annotations

import ctypes

import pytest
import torch

from block_sparse_gqa_min_b200 import sba
from tests.helpers import fill_descriptors, gpu_cache, make_case, params_of, small_workload

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("scorer", ["quest", "gate"])
def test_static_scratch_matches_caller_workspace(scorer):
    w = small_workload(d=128, H_q=8, H_kv=2, b=64, len_lo=3000, len_hi=9000, B=3, n_budget=7, n_local=2,
                       paged=True, scorer=scorer, dg=128)
    lay, li = make_case(w, seed=11)
    c = gpu_cache(w, lay, li)
    fill_descriptors(c, w, li)
    p = params_of(w)
    bufs = sba.alloc_step(c, p)
    assert sba.sba_workspace_size(c, p) <= sba.sba_static_scratch_bytes()
    q = li.q.cuda()
    for _ in range(2):  # the static scratch carries the previous call's contents into the next
        sba.sba_score_select(c, q, p, bufs.sel_idx, bufs.sel_cnt, bufs.gate_bias, bufs.ws)
        sel = torch.full_like(bufs.sel_idx, -1)
        cnt = torch.zeros_like(bufs.sel_cnt)
        gb = torch.zeros_like(bufs.gate_bias) if bufs.gate_bias is not None else None
        sba.sba_score_select_static(c, q, p, sel, cnt, gb)
        torch.cuda.synchronize()
        assert torch.equal(cnt, bufs.sel_cnt)
        for s in range(w.B):
            for h in range(w.H_kv):
                n = int(cnt[s, h])
                assert torch.equal(sel[s, h, :n], bufs.sel_idx[s, h, :n])
                if gb is not None:
                    torch.testing.assert_close(gb[s, h * w.G:(h + 1) * w.G, :n],
                                               bufs.gate_bias[s, h * w.G:(h + 1) * w.G, :n], rtol=0, atol=5e-5)
    assert int(c.status.item()) == 0


def test_static_scratch_rejects_problems_above_its_size():
    lib = sba.load()
    big = sba.sba_cache(k=0x1000, v=0x2000, block_table=None, seq_lens=0x3000, B=64, H_q=64, H_kv=8, d=128, b=64,
                        max_blocks=8192, num_pages=64 * 8192, max_len=8192 * 64, desc=0x4000, kg=None, status=None)
    p = sba.select_params(32, 2, 16, 0, 0, sba.SBA_SCORER_QUEST)
    assert lib.sba_workspace_size(ctypes.byref(big), ctypes.byref(p)) > lib.sba_static_scratch_bytes()
    rc = lib.sba_score_select_static(ctypes.byref(big), 0x5000, ctypes.byref(p), 0x6000, 0x7000, None, 64, None)
    assert rc == sba.SBA_ERR_WORKSPACE
