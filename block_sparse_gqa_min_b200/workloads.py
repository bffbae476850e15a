"""Seeded synthetic decode workloads (inputs only; none of the method's arithmetic).

The pages measure on real models and benchmark suites (AIME, MATH500, GPQA,
LongBench, RULER, ...) that are not available here; these generators stand in
for them with the SHAPES of the pages' models and the value distributions
stated per workload below.  Every tensor is drawn from a seeded torch
generator on the requested device, so the GPU path and the CPU oracle read the
same bits (the oracle gets a host copy).

Workloads (one decode step of every layer):
  tiny            1 seq, 8 Q / 2 KV heads, d 128, len 4096, b 64, budget 16
                  blocks incl. 2 local; Q,K,V ~ N(0,1); 4 "hot" blocks whose keys
                  are 0.5*mean(q of the group) + N(0,1); Quest scorer.
  qwen3_4b        36 layers x 32 Q / 8 KV heads, len 32768, b 64, budget 64
                  blocks, 2 local, min 16; K,V ~ N(0,1) x LogNormal(0,0.5)
                  per (layer, kv head, channel); Quest scorer.
  r1_7b_256k      28 layers x 28 Q / 4 KV heads (GQA 7), len 262144, b 128,
                  sparsity p = 0.95 (keep 5/100 of the blocks, rounded up),
                  4 local, min 16; N(0,1); Quest; one token appended per
                  step and, every f = 32 steps, the rectification pass of the
                  last 32 tokens (their queries, keys and values ~ N(0,1)).
  paged_b8        batch 8, 36 layers x 32/8 heads, lengths ~ U[32768, 65536],
                  64-token pages at a seed-shuffled permutation of physical
                  slots through a block table, budget 32 blocks (2048 tokens),
                  2 local, min 16; N(0,1); Quest.
  qwen3_14b_gate  40 layers x 40 Q / 8 KV heads (GQA 5), len 524288, b 64,
                  budget 32 blocks, 2 local, min 16; N(0,1); pooled
                  [max,min,avg] gate with random fp32 Wk (384->128) and Wq
                  (128->128) ~ N(0, 1/fan_in); SAS log-gate on the logits.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import List, Optional

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H_q: int
    H_kv: int
    d: int
    b: int
    layers: int
    len_lo: int
    len_hi: int                 # lengths ~ U[len_lo, len_hi] (equal = fixed)
    n_budget: int = 0
    n_local: int = 2
    n_min: int = 0
    keep_num: int = 0           # sparsity budget: keep ceil(N*keep_num/keep_den)
    keep_den: int = 0
    scorer: str = "quest"       # "quest" | "gate"
    paged: bool = False         # shuffled physical pages through a block table
    hot_blocks: int = 0
    channel_scale_sigma: float = 0.0
    append_tokens: int = 1      # tokens re-appended per step (rectification window)
    dg: int = 128               # gate width
    gate_position: str = "inner"  # gate scorer: "inner" (log g in the logits), "outer" (g on V), "off"
    gate_act: str = "softmax"     # gate scorer: "softmax", "sigmoid" or "raw"
    rectify_every: int = 0        # f: a dense rectification pass of the last f tokens every f steps

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv

    @property
    def max_len(self) -> int:
        return self.len_hi

    @property
    def max_blocks(self) -> int:
        return (self.len_hi + self.b - 1) // self.b

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, H_q=8, H_kv=2, d=128, b=64, layers=1, len_lo=4096, len_hi=4096,
                     n_budget=16, n_local=2, n_min=0, hot_blocks=4),
    "qwen3_4b": Workload("qwen3_4b", B=1, H_q=32, H_kv=8, d=128, b=64, layers=36, len_lo=32768,
                         len_hi=32768, n_budget=64, n_local=2, n_min=16, channel_scale_sigma=0.5),
    "r1_7b_256k": Workload("r1_7b_256k", B=1, H_q=28, H_kv=4, d=128, b=128, layers=28,
                           len_lo=262144, len_hi=262144, n_local=4, n_min=16, keep_num=5,
                           keep_den=100, rectify_every=32),
    "paged_b8": Workload("paged_b8", B=8, H_q=32, H_kv=8, d=128, b=64, layers=36, len_lo=32768,
                         len_hi=65536, n_budget=32, n_local=2, n_min=16, paged=True),
    "qwen3_14b_gate": Workload("qwen3_14b_gate", B=1, H_q=40, H_kv=8, d=128, b=64, layers=40,
                               len_lo=524288, len_hi=524288, n_budget=32, n_local=2, n_min=16,
                               scorer="gate"),
}
ORDER = ["tiny", "qwen3_4b", "r1_7b_256k", "paged_b8", "qwen3_14b_gate"]


@dataclass
class Layout:
    """Sequence lengths and the logical->physical page map shared by all layers."""

    seq_lens: torch.Tensor                 # int32 [B]
    block_table: Optional[torch.Tensor]    # int32 [B][max_blocks] or None
    num_pages: int
    max_blocks: int


@dataclass
class LayerInputs:
    q: torch.Tensor                 # bf16 [B][H_q][d]
    k: torch.Tensor                 # bf16 [num_pages][H_kv][b][d]
    v: torch.Tensor                 # bf16 [num_pages][H_kv][b][d]
    k_new: torch.Tensor             # bf16 [B][append_tokens][H_kv][d]
    v_new: torch.Tensor
    Wq: Optional[torch.Tensor] = None   # fp32 [dg][d]
    Wk: Optional[torch.Tensor] = None   # fp32 [dg][3d]
    hot: List[int] = field(default_factory=list)


def make_generator(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn_pages(num_pages: int, w: Workload, g: torch.Generator, dev, sc) -> torch.Tensor:
    """bf16 [num_pages][H_kv][b][d] ~ N(0,1) (times the per-channel scale, then rounded)."""
    if sc is None:
        return torch.randn((num_pages, w.H_kv, w.b, w.d), generator=g, device=dev, dtype=torch.bfloat16)
    out = torch.empty((num_pages, w.H_kv, w.b, w.d), device=dev, dtype=torch.bfloat16)
    step = 2048
    for p0 in range(0, num_pages, step):
        n = min(step, num_pages - p0)
        x = torch.randn((n, w.H_kv, w.b, w.d), generator=g, device=dev, dtype=torch.float32)
        out[p0:p0 + n] = (x * sc[None, :, None, :]).to(torch.bfloat16)
    return out


def make_layout(w: Workload, seed: int, device="cpu") -> Layout:
    """Lengths ~ U[len_lo, len_hi] (seeded ints) and, when paged, a seeded
    random permutation of physical page slots.  Block-table entries past a
    sequence's last block are -1 (never read)."""
    g = make_generator("cpu", seed * 7919 + 17)
    if w.len_lo == w.len_hi:
        lens = torch.full((w.B,), w.len_lo, dtype=torch.int32)
    else:
        lens = torch.randint(w.len_lo, w.len_hi + 1, (w.B,), generator=g, dtype=torch.int64).to(torch.int32)
    mb = w.max_blocks
    if w.paged:
        nblk = [(int(x) + w.b - 1) // w.b for x in lens]
        num_pages = int(sum(nblk))
        perm = torch.randperm(num_pages, generator=g).to(torch.int32)
        bt = torch.full((w.B, mb), -1, dtype=torch.int32)
        off = 0
        for s, n in enumerate(nblk):
            bt[s, :n] = perm[off:off + n]
            off += n
        return Layout(lens.to(device), bt.to(device), num_pages, mb)
    return Layout(lens.to(device), None, w.B * mb, mb)


def make_layer(w: Workload, lay: Layout, seed: int, layer: int, device="cpu") -> LayerInputs:
    """Synthetic inputs of one layer.  K/V are drawn page by page; pages are
    i.i.d., so drawing in physical order is the same law as drawing in logical
    order and permuting."""
    dev = torch.device(device)
    g = make_generator(dev, seed * 1_000_003 + layer * 101 + 1)
    q = torch.randn((w.B, w.H_q, w.d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    sc = None
    if w.channel_scale_sigma > 0:
        # one scale per (layer, kv head, channel), on K and V before bf16 rounding
        sc = torch.exp(w.channel_scale_sigma *
                       torch.randn((w.H_kv, w.d), generator=g, device=dev, dtype=torch.float32))
    k = _randn_pages(lay.num_pages, w, g, dev, sc)
    v = _randn_pages(lay.num_pages, w, g, dev, sc)
    kn = torch.randn((w.B, w.append_tokens, w.H_kv, w.d), generator=g, device=dev, dtype=torch.float32)
    vn = torch.randn((w.B, w.append_tokens, w.H_kv, w.d), generator=g, device=dev, dtype=torch.float32)
    if sc is not None:
        kn = kn * sc[None, None]
        vn = vn * sc[None, None]
    hot: List[int] = []
    if w.hot_blocks > 0:
        # hot blocks: keys = 0.5 * (mean of the group's query heads) + N(0,1)
        hg = make_generator("cpu", seed * 31 + layer)
        for s in range(w.B):
            n = (int(lay.seq_lens[s]) + w.b - 1) // w.b
            cand = max(0, n - w.n_local)
            pick = torch.randperm(cand, generator=hg)[: w.hot_blocks].tolist() if cand else []
            hot = sorted(pick)
            qm = q[s].float().view(w.H_kv, w.G, w.d).mean(dim=1)  # [H_kv][d]
            for j in pick:
                page = int(lay.block_table[s, j]) if lay.block_table is not None else s * lay.max_blocks + j
                noise = torch.randn((w.H_kv, w.b, w.d), generator=g, device=dev, dtype=torch.float32)
                k[page] = (0.5 * qm[:, None, :] + noise).to(torch.bfloat16)
    out = LayerInputs(q, k, v, kn.to(torch.bfloat16), vn.to(torch.bfloat16), hot=hot)
    if w.scorer == "gate":
        out.Wq = torch.randn((w.dg, w.d), generator=g, device=dev, dtype=torch.float32) / math.sqrt(w.d)
        out.Wk = torch.randn((w.dg, 3 * w.d), generator=g, device=dev, dtype=torch.float32) / math.sqrt(3 * w.d)
    return out


@dataclass
class RectInputs:
    q: torch.Tensor                 # bf16 [B][f][H_q][d]: the window's query tokens
    k_new: torch.Tensor             # bf16 [B][f][H_kv][d]: their re-encoded keys and values
    v_new: torch.Tensor


def make_rect_inputs(w: Workload, seed: int, layer: int, device="cpu") -> RectInputs:
    """Synthetic inputs of one layer's rectification pass (f = w.rectify_every tokens),
    all ~ N(0,1) in bf16 from their own seeded generator."""
    f = w.rectify_every
    dev = torch.device(device)
    g = make_generator(dev, seed * 1_000_033 + layer * 103 + 7)
    q = torch.randn((w.B, f, w.H_q, w.d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    kn = torch.randn((w.B, f, w.H_kv, w.d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    vn = torch.randn((w.B, f, w.H_kv, w.d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    return RectInputs(q, kn, vn)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Host numpy uint16 view of a bf16 tensor's bits."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)

