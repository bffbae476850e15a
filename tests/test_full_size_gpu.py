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
