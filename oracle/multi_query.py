"""Several query tokens per sequence sharing one block selection, on the CPU in
fp64: TEST INFRASTRUCTURE ONLY.

Only tests import this module; the CUDA library has no counterpart yet (this is
a next step of the build).

Sources (page title, section): "Rectified Sparse Attention for Efficient
Long-Sequence Generation", Summary (after every f generated tokens those tokens
are re-encoded in one parallel dense pass; all query heads of a GQA group share
one block selection) and Key points (f in {16, 32, 64, 128}; the comparison with
sparse-KV self-speculative decoding, which verifies several draft tokens at
once).

Readings where the pages are silent (also listed in the design notes):
  * the M query tokens of a sequence sit at the last M positions of its cache,
    len-M .. len-1, whose keys and values are already written;
  * the group shares ONE selection for all M tokens, ranked by the group score
    summed over the G heads and the M tokens (the M tokens act as extra heads of
    the group);
  * token i attends causally: only to positions t <= len - M + i;
  * the dense rectification pass is the same computation with every block
    selected.

The scores, the top-n rule and the per-token attention are the main oracle's
(``oracle.quest_scores``, ``oracle.select``, ``oracle.attend``), each pinned by
the main pin suite; this module only sums, truncates and loops.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

from . import Cache, attend, quest_scores, select


def _truncated(c: Cache, seq_lens: np.ndarray) -> Cache:
    """The same pages seen with other lengths (the causal horizon of one token)."""
    return Cache(c.k, c.v, c.block_table, np.asarray(seq_lens, dtype=np.int32), H_q=c.H_q,
                 max_blocks=c.max_blocks)


def decode_multi(c: Cache, q: np.ndarray, *, scale: float, n_budget: int, n_local: int, n_min: int,
                 keep_num: int = 0, keep_den: int = 0, dense: bool = False, n_max: Optional[int] = None,
                 sel=None):
    """q: bf16 bits [B][M][H_q][d].  Returns (score [B][H_kv][max_blocks], sel_idx, sel_cnt,
    out [B][M][H_q][d], lse [B][M][H_q]); dense=True selects every block (the
    rectification pass); sel = (sel_idx, sel_cnt) replaces the top-n selection by a
    given one (used to re-run a near-tie case)."""
    q = np.asarray(q, dtype=np.uint16)
    B, M = q.shape[0], q.shape[1]
    score = np.zeros((c.B, c.H_kv, c.max_blocks))
    for i in range(M):
        score += quest_scores(c, np.ascontiguousarray(q[:, i]))
    if n_max is None:
        n_max = max(1, c.max_blocks)
    if dense:
        N = c.n_blocks()
        sel_idx = np.full((c.B, c.H_kv, n_max), -1, dtype=np.int32)
        sel_cnt = np.zeros((c.B, c.H_kv), dtype=np.int32)
        for s in range(c.B):
            sel_idx[s, :, : N[s]] = np.arange(N[s], dtype=np.int32)
            sel_cnt[s, :] = N[s]
    elif sel is not None:
        sel_idx, sel_cnt = (np.asarray(x, dtype=np.int32) for x in sel)
    else:
        sel_idx, sel_cnt = select(score, c.seq_lens, c.b, n_budget, n_local, n_min, keep_num, keep_den, n_max)
    out = np.zeros((B, M, c.H_q, c.d))
    lse = np.zeros((B, M, c.H_q))
    for i in range(M):
        horizon = np.maximum(c.seq_lens.astype(np.int64) - M + i + 1, 0)
        o, l = attend(_truncated(c, horizon), np.ascontiguousarray(q[:, i]), sel_idx, sel_cnt, scale)
        out[:, i] = o
        lse[:, i] = l
    return score, sel_idx, sel_cnt, out, lse
