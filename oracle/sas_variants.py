"""SAS gate variants on the CPU, in fp64: TEST INFRASTRUCTURE ONLY.

Only tests import this module; nothing on the product path does, and the CUDA
library has no counterpart yet (the variants are a next step of the build).

Source: "SAS: Simple Attention Sparsification via End-to-End Optimization of
Context Ranking", Method.  The context is the always-kept current block B0
(gate g0 = 1) and the C historical blocks B1..BC; the selector's scores s give
positive gates g = phi(s) on the historical blocks.  Two gate positions:
inner, o = softmax(q K^T + log g) V, and outer, o = softmax(q K^T) (g . V)
(each token's value scaled by its block's gate); three activations phi:
softmax (normalised over the C blocks), sigmoid (each block on its own) and
unnormalised logit injection.

Readings where the page is silent (also listed in the design notes):
  * s is the gate logit of the main gate scorer, u = (Wq q).(Wk pooled)/sqrt(dg)
    ("SeerAttention-R", abstract: the gate scores blocks from the decode query);
  * unnormalised logit injection adds s itself to the logits: log g = s;
  * the group shares one selection ranked by the sum of its heads' gates
    sum_h g_h (as for the softmax gate), and the current block is always kept;
  * with the outer position the logits carry no gate and lse is that of the
    ungated logits.

Every step is written out with plain numpy loops over the selected tokens; the
descriptors and the top-n selection are the main oracle's (``oracle.gate_desc``,
``oracle.select``), whose pins cover them.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

from . import Cache, Decoded, gate_desc, select

ACTIVATIONS = ("softmax", "sigmoid", "raw")
POSITIONS = ("inner", "outer")


def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def gate_logits(c: Cache, q: np.ndarray, Wq: np.ndarray, Wk: np.ndarray) -> np.ndarray:
    """u [B][H_q][max_blocks] for the historical blocks j < N-1 (NaN elsewhere):
    u_j = (Wq q) . kg_j / sqrt(dg), kg the stored gate key of block j."""
    _, kg = gate_desc(c, Wk)
    Wq64 = np.asarray(Wq, dtype=np.float32).astype(np.float64)
    dg = Wq64.shape[0]
    qf = _bf16_to_f64(np.asarray(q, dtype=np.uint16))
    u = np.full((c.B, c.H_q, c.max_blocks), np.nan)
    N = c.n_blocks()
    for s in range(c.B):
        for qh in range(c.H_q):
            h = qh // c.G
            qp = Wq64 @ qf[s, qh]
            for j in range(int(N[s]) - 1):
                u[s, qh, j] = float(qp @ kg[s, j, h]) / math.sqrt(dg)
    return u


def log_gates(u: np.ndarray, activation: str) -> np.ndarray:
    """log g over the C historical blocks of one head (u: [C])."""
    u = np.asarray(u, dtype=np.float64)
    if u.size == 0:
        return u.copy()
    if activation == "softmax":
        m = u.max()
        return u - (m + math.log(np.exp(u - m).sum()))
    if activation == "sigmoid":
        # log(1 / (1 + e^-u)), written without overflow on either side
        return np.where(u >= 0, -np.log1p(np.exp(-np.abs(u))), u - np.log1p(np.exp(-np.abs(u))))
    if activation == "raw":
        return u.copy()
    raise ValueError(activation)


def decode_variant(c: Cache, q: np.ndarray, Wq: np.ndarray, Wk: np.ndarray, *, scale: float, n_budget: int,
                   n_local: int, n_min: int, activation: str = "softmax", position: str = "inner",
                   n_max: Optional[int] = None, sel=None) -> Decoded:
    """One decode step with a SAS gate variant: gates, group scores, selection
    (current block always kept), attention with the gate inside or outside the
    softmax.  Returns the main oracle's Decoded record (logg = log g, 0 on B0).
    sel = (sel_idx, sel_cnt) replaces the top-n selection by a given one (the
    attention is then over those blocks; used to re-run a near-tie case)."""
    if position not in POSITIONS:
        raise ValueError(position)
    q = np.asarray(q, dtype=np.uint16)
    u = gate_logits(c, q, Wq, Wk)
    N = c.n_blocks()
    logg = np.full((c.B, c.H_q, c.max_blocks), np.nan)
    score = np.full((c.B, c.H_kv, c.max_blocks), np.nan)
    for s in range(c.B):
        Ns = int(N[s])
        if Ns == 0:
            continue
        score[s, :, :Ns] = 0.0
        for qh in range(c.H_q):
            lg = log_gates(u[s, qh, : Ns - 1], activation)
            logg[s, qh, : Ns - 1] = lg
            logg[s, qh, Ns - 1] = 0.0           # B0: unit gate
            score[s, qh // c.G, : Ns - 1] += np.exp(lg)
    if n_max is None:
        n_max = max(1, c.max_blocks)
    if sel is None:
        sel_idx, sel_cnt = select(score, c.seq_lens, c.b, n_budget, max(n_local, 1), n_min, n_max=n_max)
    else:
        sel_idx, sel_cnt = (np.asarray(x, dtype=np.int32) for x in sel)

    qf = _bf16_to_f64(q)
    out = np.zeros((c.B, c.H_q, c.d))
    lse = np.full((c.B, c.H_q), -np.inf)
    for s in range(c.B):
        L = int(c.seq_lens[s])
        for qh in range(c.H_q):
            h = qh // c.G
            logits, gates, vals = [], [], []
            for i in range(int(sel_cnt[s, h])):
                j = int(sel_idx[s, h, i])
                page = int(c.block_table[s, j]) if c.block_table is not None else s * c.max_blocks + j
                for t in range(j * c.b, min((j + 1) * c.b, L)):
                    k = _bf16_to_f64(c.k[page, h, t % c.b])
                    lt = float(qf[s, qh] @ k) * scale
                    if position == "inner":
                        lt += logg[s, qh, j]
                    logits.append(lt)
                    gates.append(math.exp(logg[s, qh, j]))
                    vals.append(_bf16_to_f64(c.v[page, h, t % c.b]))
            if not logits:
                continue
            lg = np.array(logits)
            m = lg.max()
            w = np.exp(lg - m)
            z = w.sum()
            for t in range(len(logits)):
                g = gates[t] if position == "outer" else 1.0
                out[s, qh] += (w[t] / z) * g * vals[t]
            lse[s, qh] = m + math.log(z)
    return Decoded(score, sel_idx, sel_cnt, logg, out, lse)
