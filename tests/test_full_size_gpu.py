"""Full-size parity: each model-shaped workload at its real context length, one
sampled (middle) layer, through the fused one-launch step that bench.py times,
against the oracle run on the whole layer (selection of every group, every
output element)."""
from __future__ import annotations

import pytest
import torch

from block_sparse_gqa_min_b200 import workloads as W
from tests.test_fused_step_gpu import run_fused

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("name", ["tiny", "qwen3_4b", "r1_7b_256k", "paged_b8", "qwen3_14b_gate"])
def test_full_size_sampled_layer(name):
    w = W.WORKLOADS[name]
    lay = W.make_layout(w, 0, device="cuda")
    li = W.make_layer(w, lay, 0, w.layers // 2, device="cuda")
    r = run_fused(w, seed=0, n_app=w.append_tokens, layout=lay, layer_inputs=li)
    assert r["err"] <= 2e-3


def test_full_size_rectification_sampled_rows():
    """The R1-7B-shaped rectification pass (f = 32 at 262144 tokens, one sampled layer):
    the window's rows and the refreshed descriptors exactly, and the dense causal output
    of the first and last window token (every query head) against the oracle, each
    computed on its own causal horizon."""
    import numpy as np

    import oracle as O
    from block_sparse_gqa_min_b200 import sba
    from tests.helpers import ATOL_OUT, fill_descriptors, gpu_cache

    w = W.WORKLOADS["r1_7b_256k"]
    f = w.rectify_every
    lay = W.make_layout(w, 0, device="cuda")
    li = W.make_layer(w, lay, 0, w.layers // 2, device="cuda")
    ri = W.make_rect_inputs(w, 0, w.layers // 2, device="cuda")
    c = gpu_cache(w, lay, li)
    fill_descriptors(c, w, li)
    rg = sba.sba_multi_row_groups(c, f)
    S = max(1, 148 // (w.B * w.H_kv * rg))
    o_part = torch.empty((w.B, f, w.H_q, S, w.d), dtype=torch.float32, device="cuda")
    lse_part = torch.empty((w.B, f, w.H_q, S), dtype=torch.float32, device="cuda")
    out = torch.empty((w.B, f * w.H_q, w.d), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, f * w.H_q), dtype=torch.float32, device="cuda")
    sba.sba_rectify(c, ri.q, ri.k_new, ri.v_new, w.scale, o_part, lse_part)
    sba.sba_combine(o_part, lse_part, out, lse)
    torch.cuda.synchronize()
    assert int(c.status.item()) == 0
    L = int(lay.seq_lens[0])
    pages = [L // w.b - 1 + (1 if L % w.b else 0)]  # contiguous: page = block
    k_host = c.k.cpu()
    assert torch.equal(k_host[pages[0], :, (L - f) % w.b:(L - 1) % w.b + 1].transpose(0, 1), ri.k_new[0].cpu())
    assert torch.equal(c.v[pages[0], :, (L - f) % w.b:(L - 1) % w.b + 1].transpose(0, 1).cpu(), ri.v_new[0].cpu())
    blk = k_host[pages[0]].float()  # [H_kv][b][d], every row valid (L is a multiple of b)
    d = c.desc[pages[0]].float().cpu()
    assert torch.equal(d[:, 0], blk.amin(dim=1)) and torch.equal(d[:, 1], blk.amax(dim=1))
    oc = O.Cache(W.bf16_bits(k_host), W.bf16_bits(c.v), None, np.array([L], dtype=np.int32), H_q=w.H_q,
                 max_blocks=lay.max_blocks)
    N = (L + w.b - 1) // w.b
    got = out.view(w.B, f, w.H_q, w.d).cpu().numpy()
    for i in (0, f - 1):
        horizon = L - f + i + 1
        oci = O.Cache(oc.k, oc.v, None, np.array([horizon], dtype=np.int32), H_q=w.H_q, max_blocks=lay.max_blocks)
        Ni = (horizon + w.b - 1) // w.b
        sel = np.arange(N, dtype=np.int32)[None, None, :].repeat(w.H_kv, axis=1)
        cnt = np.full((1, w.H_kv), Ni, dtype=np.int32)
        o_ref, _ = O.attend(oci, W.bf16_bits(ri.q[:, i]), sel, cnt, w.scale)
        err = float(np.abs(got[0, i] - o_ref[0]).max())
        assert err <= ATOL_OUT, (i, err)
