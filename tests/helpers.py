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


# ---------------------------------------------------------------------------
# GPU-side helpers (used only by tests marked gpu)
# ---------------------------------------------------------------------------

ATOL_OUT = 2e-3        # attention output, max-abs (bf16 inputs, fp32 accumulation)
NEAR_TIE_REL = 1e-5    # near-tie band for selection differences


def gpu_cache(w: W.Workload, lay: W.Layout, li: W.LayerInputs, max_len=None):
    """Device tensors of one layer with zeroed descriptors and a status word."""
    from block_sparse_gqa_min_b200 import sba

    dev = torch.device("cuda")
    k, v = li.k.to(dev), li.v.to(dev)
    c = sba.Cache(
        k=k, v=v, seq_lens=lay.seq_lens.to(dev, torch.int32), H_q=w.H_q, max_blocks=lay.max_blocks,
        max_len=int(max_len if max_len is not None else lay.seq_lens.max().item()),
        block_table=None if lay.block_table is None else lay.block_table.to(dev, torch.int32),
        desc=torch.zeros((lay.num_pages, w.H_kv, 2, w.d), dtype=torch.bfloat16, device=dev)
        if w.scorer == "quest" else None,
        kg=torch.zeros((lay.num_pages, w.H_kv, w.d), dtype=torch.float32, device=dev)
        if w.scorer == "gate" else None,
        status=torch.zeros((1,), dtype=torch.int32, device=dev),
    )
    return c


def fill_descriptors(c, w: W.Workload, li: W.LayerInputs):
    from block_sparse_gqa_min_b200 import sba

    pos0 = torch.zeros((c.B,), dtype=torch.int32, device=c.k.device)
    if w.scorer == "gate":
        sba.sba_update_descriptors(c, pos0, c.max_len, li.Wq.cuda(), li.Wk.cuda())
    else:
        sba.sba_update_descriptors(c, pos0, c.max_len)


def params_of(w: W.Workload):
    from block_sparse_gqa_min_b200 import sba

    gate = w.scorer == "gate"
    pos = {"off": sba.SBA_LOG_GATE_OFF, "inner": sba.SBA_LOG_GATE_INNER, "outer": sba.SBA_LOG_GATE_OUTER}
    act = {"softmax": sba.SBA_GATE_SOFTMAX, "sigmoid": sba.SBA_GATE_SIGMOID, "raw": sba.SBA_GATE_RAW}
    return sba.select_params(w.n_budget, w.n_local, w.n_min, w.keep_num, w.keep_den,
                             sba.SBA_SCORER_GATE if gate else sba.SBA_SCORER_QUEST,
                             pos[w.gate_position] if gate else 0, act[w.gate_act] if gate else 0)


def oracle_decode(w: W.Workload, oc: O.Cache, li: W.LayerInputs, n_max=None, sel=None):
    """The oracle's whole step for workload w (the gate variants through
    oracle.sas_variants); sel = (sel_idx, sel_cnt) re-runs it on a given selection."""
    if w.scorer == "gate" and (w.gate_act != "softmax" or w.gate_position == "outer"):
        from oracle import sas_variants as V

        d = V.decode_variant(oc, W.bf16_bits(li.q), li.Wq.cpu().numpy(), li.Wk.cpu().numpy(), scale=w.scale,
                             n_budget=w.n_budget, n_local=w.n_local, n_min=w.n_min, activation=w.gate_act,
                             position=w.gate_position if w.gate_position != "off" else "inner", n_max=n_max,
                             sel=sel)
        if w.gate_position == "off":  # the gates select; the attention is plain
            o, l = O.attend(oc, W.bf16_bits(li.q), d.sel_idx, d.sel_cnt, w.scale, None)
            d = O.Decoded(d.score, d.sel_idx, d.sel_cnt, d.logg, o, l)
        return d
    kw = dict(scale=w.scale, n_budget=w.n_budget, n_local=w.n_local, n_min=w.n_min,
              keep_num=w.keep_num, keep_den=w.keep_den, scorer=w.scorer, n_max=n_max,
              log_gate=w.gate_position != "off")
    if w.scorer == "gate":
        kw.update(Wq=li.Wq.cpu().numpy(), Wk=li.Wk.cpu().numpy())
    d = O.decode(oc, W.bf16_bits(li.q), **kw)
    if sel is not None:
        bias = d.logg if (w.scorer == "gate" and w.gate_position != "off") else None
        o, l = O.attend(oc, W.bf16_bits(li.q), sel[0], sel[1], w.scale, bias)
        d = O.Decoded(d.score, np.asarray(sel[0]), np.asarray(sel[1]), d.logg, o, l)
    return d


def check_selection(ref: O.Decoded, sel_idx: np.ndarray, sel_cnt: np.ndarray, oc: O.Cache, w: W.Workload):
    """Bit-exact block sets, or differences confined to near-ties of the oracle's
    own scores (|s - theta| <= 1e-5 |theta|, theta = score of the last block the
    oracle admitted).  Returns the number of (sequence, group) near-tie events."""
    events = 0
    L_eff = max(w.n_local, 1) if w.scorer == "gate" else w.n_local
    for s in range(oc.B):
        N = int(oc.n_blocks()[s])
        L = min(L_eff, N)
        for h in range(oc.H_kv):
            n_ref = int(ref.sel_cnt[s, h])
            assert int(sel_cnt[s, h]) == n_ref, (s, h, int(sel_cnt[s, h]), n_ref)
            a = set(ref.sel_idx[s, h, :n_ref].tolist())
            b = sel_idx[s, h, :n_ref].tolist()
            assert b == sorted(b), "selection must ascend"
            if a == set(b):
                continue
            events += 1
            sc = ref.score[s, h, : N - L].astype(np.float32).astype(np.float64)
            admitted = [j for j in a if j < N - L]
            theta = min(sc[j] for j in admitted)
            diff = a.symmetric_difference(b)
            for j in diff:
                assert j < N - L, "a local block differs"
                assert abs(sc[j] - theta) <= NEAR_TIE_REL * abs(theta), (s, h, j, sc[j], theta)
    return events
