"""Shared test helpers: small seeded caches for the oracle and the GPU path."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from block_sparse_gqa_min_b200 import workloads as W


def small_workload(**kw) -> W.Workload:
    base = dict(name="t", B=1, H_q=4, H_kv=2, d=8, b=4, layers=1, len_lo=23, len_hi=23,
                n_budget=3, n_local=1, n_min=0)
    base.update(kw)
    return W.Workload(**base)


def oracle_cache(w: W.Workload, lay: W.Layout, li: W.LayerInputs) -> O.Cache:
    bt = None if lay.block_table is None else lay.block_table.cpu().numpy()
    return O.Cache(W.bf16_bits(li.k), W.bf16_bits(li.v), bt, lay.seq_lens.cpu().numpy(),
                   H_q=w.H_q, max_blocks=lay.max_blocks)


def make_case(w: W.Workload, seed: int = 0, device: str = "cpu"):
    lay = W.make_layout(w, seed, device=device)
    li = W.make_layer(w, lay, seed, 0, device=device)
    return lay, li


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def gather_tokens(c: O.Cache, s: int, h: int, which: str = "k") -> np.ndarray:
    """All valid tokens [len][d] (fp64) of sequence s, kv head h, in logical order."""
    arr = c.k if which == "k" else c.v
    L = int(c.seq_lens[s])
    rows = []
    for t in range(L):
        j = t // c.b
        p = int(c.block_table[s, j]) if c.block_table is not None else s * c.max_blocks + j
        rows.append(bf16_to_f64(arr[p, h, t % c.b]))
    return np.array(rows).reshape(L, c.d)
