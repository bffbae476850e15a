"""Decode-step benchmark: µs/step and achieved HBM GB/s of the block-sparse GQA
decode path on synthetic workloads shaped like the pages' models.

One step = for every layer: append the step's new K/V tokens, refresh the
descriptors of the touched blocks, score + select, sparse decode, combine --
all through libsba's C ABI, captured once in a CUDA graph and replayed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Multi-GPU (torchrun, one process per GPU): every rank decodes its own
independent batch of the same shape (weak scaling); no collective touches the
data path; the step time is the max over ranks.

Counted bytes per layer and step (what the method must read): the selected
K+V blocks (n_sel * b * d * 2 tensors * 2 B per KV head and sequence) plus the
block descriptors (N * 512 B per KV head and sequence).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-decode µs/step and achieved HBM GB/s (% of B200 roofline) vs context"
DEFAULT_WORKLOAD = "qwen3_4b"
DESC_BYTES = 512  # Quest bf16 min+max, or gate fp32 key, per block and KV head


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (0 = workload's)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--path", default="fused", choices=["fused", "separate"],
                    help="fused: one sba_decode_step launch per layer; separate: the five single-step calls")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_seed(seed: int, rank: int) -> int:
    """Every rank decodes its own independent batch (weak scaling)."""
    return seed + 1000 * rank


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """Step time of the job = the slowest rank's (max-reduce of one scalar)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist

    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(step_bytes_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: bytes every rank processed / the max step time."""
    return step_bytes_per_rank * world / (ms_max * 1e-3) / 1e9


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# sources of the fused step kernel: a recorded ncu traffic figure is valid only while they are unchanged
KERNEL_SOURCES = {
    "decode_step": ["fused_step.cu", "decode_tile.cuh", "select.cuh", "common.cuh", "launch.cuh"],
}


def kernel_source_hash(kernel: str) -> str:
    import hashlib

    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, []):
        with open(os.path.join(ROOT, "block_sparse_gqa_min_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch (read + write) from the committed ncu summary of this
    kernel and workload, or None when there is none or the kernel changed since."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    fields = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    if fields.get("source_sha256") != kernel_source_hash(kernel):
        return None
    try:
        return int(float(fields["dram_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


def counted_bytes(w, seq_lens, n_sel_of):
    """Counted bytes of one layer for the given lengths."""
    tot = 0
    for L in seq_lens:
        N = (int(L) + w.b - 1) // w.b
        tot += n_sel_of(N) * w.b * w.d * 2 * 2 * w.H_kv + N * w.H_kv * DESC_BYTES
    return tot


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# native arm
# ---------------------------------------------------------------------------

def build_layers(w, lay, seed, n_layers, dev):
    import torch

    from block_sparse_gqa_min_b200 import sba
    from block_sparse_gqa_min_b200 import workloads as W

    gate = w.scorer == "gate"
    p = sba.select_params(w.n_budget, w.n_local, w.n_min, w.keep_num, w.keep_den,
                          sba.SBA_SCORER_GATE if gate else sba.SBA_SCORER_QUEST)
    layers = []
    max_len = int(lay.seq_lens.max().item())
    ws = None
    for l in range(n_layers):
        li = W.make_layer(w, lay, seed, l, device=dev)
        c = sba.Cache(
            k=li.k, v=li.v, seq_lens=lay.seq_lens, H_q=w.H_q, max_blocks=lay.max_blocks, max_len=max_len,
            block_table=lay.block_table,
            desc=None if gate else torch.zeros((lay.num_pages, w.H_kv, 2, w.d), dtype=torch.bfloat16, device=dev),
            kg=torch.zeros((lay.num_pages, w.H_kv, w.d), dtype=torch.float32, device=dev) if gate else None,
            status=torch.zeros((1,), dtype=torch.int32, device=dev))
        pos0 = torch.zeros((w.B,), dtype=torch.int32, device=dev)
        if gate:
            sba.sba_update_descriptors(c, pos0, max_len, li.Wq, li.Wk)
        else:
            sba.sba_update_descriptors(c, pos0, max_len)
        bufs = sba.alloc_step(c, p)
        if ws is None:
            ws = bufs.ws
        bufs.ws = ws  # calls are stream-ordered, so layers share one workspace
        A = None
        if gate:
            A = torch.empty((w.d, 3 * w.d), dtype=torch.float32, device=dev)
            sba.sba_fold_gate(li.Wq, li.Wk, A)
        layers.append(dict(c=c, li=li, bufs=bufs, A=A))
    # positions of the step's re-appended tokens: the last `append_tokens` positions
    pos = (lay.seq_lens - w.append_tokens).clamp(min=0).to(torch.int32)
    torch.cuda.synchronize()
    return layers, p, pos


def layer_step(w, L, p, pos, q=None, k_new=None, v_new=None, path="fused", out=None):
    from block_sparse_gqa_min_b200 import sba

    c, li, bufs = L["c"], L["li"], L["bufs"]
    q = li.q if q is None else q
    if path == "fused":
        sba.sba_decode_step(c, q, p, w.scale, bufs.out if out is None else out, bufs.lse,
                            k_new=li.k_new if k_new is None else k_new,
                            v_new=li.v_new if v_new is None else v_new, pos_start=pos, gate_A=L["A"],
                            sel_idx=bufs.sel_idx, sel_cnt=bufs.sel_cnt, gate_bias=bufs.gate_bias)
        return
    sba.sba_append_kv(c, li.k_new if k_new is None else k_new, li.v_new if v_new is None else v_new, pos)
    if w.scorer == "gate":
        sba.sba_update_descriptors(c, pos, w.append_tokens, li.Wq, li.Wk)
    else:
        sba.sba_update_descriptors(c, pos, w.append_tokens)
    sba.decode_step(c, q, p, bufs, w.scale)


KERNELS_PER_LAYER = {"fused": 1, "separate": 5}  # separate: append, update, score+select, decode, combine


def native(args, rank, world, local):
    import torch
    import torch.distributed as dist

    from block_sparse_gqa_min_b200 import sba
    from block_sparse_gqa_min_b200 import workloads as W

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    sba.load()
    w = W.WORKLOADS[args.workload]
    n_layers = args.layers or w.layers
    seed = rank_seed(args.seed, rank)
    lay = W.make_layout(w, seed, device=dev)
    layers, p, pos = build_layers(w, lay, seed, n_layers, dev)
    n_max = layers[0]["bufs"].sel_idx.shape[-1]
    splits = layers[0]["bufs"].lse_part.shape[-1]
    lens = lay.seq_lens.cpu().tolist()
    per_layer = counted_bytes(w, lens, lambda N: sba.sba_num_selected(N, p))
    step_bytes = per_layer * n_layers
    kv_bytes_layer = sum(sba.sba_num_selected((L + w.b - 1) // w.b, p) * w.b * w.d * 4 * w.H_kv for L in lens)
    desc_bytes_layer = sum(((L + w.b - 1) // w.b) * w.H_kv * DESC_BYTES for L in lens)

    def step():
        for L in layers:
            layer_step(w, L, p, pos, path=args.path)

    # capture one step in a CUDA graph
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    torch.cuda.synchronize()

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    footprint = step_bytes
    flush = footprint < 4 * l2
    flush_buf = torch.empty((512 * 1024 * 1024 // 4,), dtype=torch.float32, device=dev) if flush else None

    for _ in range(max(args.warmup, 3)):
        graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps + 2)]
    if flush:
        total_ms = 0.0
        for i in range(args.steps):
            flush_buf.fill_(float(i))
            ev[2 * i].record()
            graph.replay()
            ev[2 * i + 1].record()
        torch.cuda.synchronize()
        total_ms = sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(args.steps))
    else:
        ev[0].record()
        for _ in range(args.steps):
            graph.replay()
        ev[1].record()
        torch.cuda.synchronize()
        total_ms = ev[0].elapsed_time(ev[1])
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    ms_max = max_over_ranks(total_ms / args.steps, world, dev)
    value = job_gbs(step_bytes, world, ms_max)

    # ---- per-launch durations, measured live on the launching stream ----
    # launches are queued behind a sleep kernel so that host-side gaps between
    # them do not appear in the device-side event intervals
    names = ["decode_step"] if args.path == "fused" else ["append_kv", "update_descriptors", "score_select",
                                                          "sparse_decode", "combine"]
    kt = {k: [] for k in names}
    for _ in range(3):
        torch.cuda._sleep(int(2e8))
        rec = []
        for L in layers:
            c, li, bufs = L["c"], L["li"], L["bufs"]
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
            ev[0].record()
            if args.path == "fused":
                layer_step(w, L, p, pos, path="fused")
                ev[1].record()
            else:
                sba.sba_append_kv(c, li.k_new, li.v_new, pos)
                ev[1].record()
                if w.scorer == "gate":
                    sba.sba_update_descriptors(c, pos, w.append_tokens, li.Wq, li.Wk)
                else:
                    sba.sba_update_descriptors(c, pos, w.append_tokens)
                ev[2].record()
                sba.sba_score_select(c, li.q, p, bufs.sel_idx, bufs.sel_cnt, bufs.gate_bias, bufs.ws)
                ev[3].record()
                sba.sba_sparse_decode(c, li.q, bufs.sel_idx, bufs.sel_cnt, bufs.gate_bias, w.scale, bufs.o_part,
                                      bufs.lse_part)
                ev[4].record()
                sba.sba_combine(bufs.o_part, bufs.lse_part, bufs.out, bufs.lse)
                ev[5].record()
            rec.append(ev)
        torch.cuda.synchronize()
        for ev in rec:
            for i, k in enumerate(names):
                kt[k].append(ev[i].elapsed_time(ev[i + 1]))
    kmean = {k: statistics.mean(v) for k, v in kt.items()}
    if args.path == "fused":
        alg = {"decode_step": per_layer}
    else:
        alg = {"sparse_decode": kv_bytes_layer, "score_select": desc_bytes_layer}
    dom = max(alg, key=lambda k: kmean[k])
    hbm, peak_kind = peaks()
    achieved = alg[dom] / (kmean[dom] * 1e-3) / 1e9
    roof = {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "peak_source": peak_kind,
            "alg_bytes_per_launch": alg[dom], "launch_us": round(kmean[dom] * 1e3, 3),
            "traffic": recorded_traffic(dom, w.name),
            "other_kernels_us": {k: round(v * 1e3, 3) for k, v in kmean.items() if k != dom},
            "step_frac": round(step_bytes / (ms_max * 1e-3) / 1e9 / hbm, 4)}

    # ---- e2e: host buffers, copies inside the timed region ----
    e2e = None
    if not args.no_e2e:
        # a step's inputs of every layer in one pinned host buffer per tensor, every layer's output
        # back in one copy: one host-to-device copy per input tensor and one device-to-host copy
        def stacked(ts):
            h = torch.empty((len(ts),) + tuple(ts[0].shape), dtype=ts[0].dtype).pin_memory()
            for i, t in enumerate(ts):
                h[i].copy_(t)
            return h, torch.empty(h.shape, dtype=h.dtype, device=dev)
        qh, qd = stacked([L["li"].q for L in layers])
        kh, kd = stacked([L["li"].k_new for L in layers])
        vh, vd = stacked([L["li"].v_new for L in layers])
        out0 = layers[0]["bufs"].out
        od = torch.empty((len(layers),) + tuple(out0.shape), dtype=out0.dtype, device=dev)
        oh = torch.empty(od.shape, dtype=od.dtype).pin_memory()
        h2d = sum(x.numel() * x.element_size() for x in (qh, kh, vh))
        d2h = oh.numel() * oh.element_size()

        def e2e_step():
            qd.copy_(qh, non_blocking=True)
            kd.copy_(kh, non_blocking=True)
            vd.copy_(vh, non_blocking=True)
            for i, L in enumerate(layers):
                if args.path == "fused":
                    layer_step(w, L, p, pos, q=qd[i], k_new=kd[i], v_new=vd[i], path="fused", out=od[i])
                else:
                    layer_step(w, L, p, pos, q=qd[i], k_new=kd[i], v_new=vd[i], path=args.path)
                    od[i].copy_(L["bufs"].out)
            oh.copy_(od, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, min(args.steps, 20))
        e0.record()
        for _ in range(n_e2e):
            e2e_step()
        e1.record()
        torch.cuda.synchronize()
        t_e2e = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world, dev)
        e2e = {"value": round(job_gbs(step_bytes, world, t_e2e), 1), "unit": "GB/s",
               "ms_per_step": round(t_e2e, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "api": ("eager C-ABI call per layer; q, k_new, v_new of all layers from one pinned host buffer "
                       "each (one copy per tensor per step), every layer's fp32 output back in one copy")}

    status = [int(L["c"].status.item()) for L in layers]
    if any(status):
        raise RuntimeError(f"device status bits set: {status}")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, lay, layers, p, args.cpu_seconds)

    out = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(args.warmup, 3),
        "ms_per_step": round(ms_max, 4),
        "us_per_step": round(ms_max * 1e3, 1),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; shapes and distributions of the workload, no model weights)",
        "config": {
            "workload": w.name, "batch": w.B, "layers": n_layers, "H_q": w.H_q, "H_kv": w.H_kv, "d": w.d,
            "block": w.b, "context": [min(lens), max(lens)], "blocks_selected_per_group": n_max,
            "scorer": w.scorer, "paged": w.paged, "append_tokens_per_step": w.append_tokens,
            "num_splits": splits, "cluster_ctas": sba.sba_decode_step_cluster(layers[0]["c"], p),
            "counted_bytes_per_step": step_bytes,
            "kv_bytes_per_layer": kv_bytes_layer, "desc_bytes_per_layer": desc_bytes_layer,
            "l2": (f"L2 flushed between steps (512 MB write, outside the timed events); step footprint "
                   f"{footprint / 1e6:.0f} MB" if flush else
                   f"inputs larger than L2: {footprint / 1e6:.0f} MB per step vs {l2 / 1e6:.0f} MB L2"),
            "graph": "one CUDA graph per step, programmatic dependent launch between kernels",
            "path": ("one fused sba_decode_step launch per layer (thread-block clusters)" if args.path == "fused"
                     else "five C-ABI calls per layer"),
            "parallelism": f"replicas x{world} (independent batches, no collective)",
        },
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": KERNELS_PER_LAYER[args.path] * n_layers * args.steps,
        "clocks": clk,
    }
    del graph
    return out


# ---------------------------------------------------------------------------
# CPU oracle (timed baseline and the --impl reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(w, lay_cpu, layer_inputs_fn, n_layers, budget_s, p_num_sel):
    """Run the oracle's whole step (descriptors -> scores -> selection ->
    attention) on evenly spaced layers until `budget_s` seconds are used."""
    import oracle as O
    from block_sparse_gqa_min_b200 import workloads as W

    order = sorted(set([0, n_layers - 1, n_layers // 2] + list(range(n_layers))), key=lambda l: (
        0 if l in (0, n_layers - 1, n_layers // 2) else 1, l))
    done, t_cpu, bytes_done = [], 0.0, 0
    lens = lay_cpu.seq_lens.tolist()
    per_layer = counted_bytes(w, lens, p_num_sel)
    for l in order:
        li = layer_inputs_fn(l)
        oc = O.Cache(W.bf16_bits(li.k), W.bf16_bits(li.v),
                     None if lay_cpu.block_table is None else lay_cpu.block_table.numpy(),
                     lay_cpu.seq_lens.numpy(), H_q=w.H_q, max_blocks=lay_cpu.max_blocks)
        kw = dict(scale=w.scale, n_budget=w.n_budget, n_local=w.n_local, n_min=w.n_min, keep_num=w.keep_num,
                  keep_den=w.keep_den, scorer=w.scorer)
        if w.scorer == "gate":
            kw.update(Wq=li.Wq.cpu().numpy(), Wk=li.Wk.cpu().numpy())
        qb = W.bf16_bits(li.q)
        t0 = time.perf_counter()
        O.decode(oc, qb, **kw)
        t_cpu += time.perf_counter() - t0
        done.append(l)
        bytes_done += per_layer
        if t_cpu >= budget_s:
            break
    return done, t_cpu, bytes_done


def cpu_baseline(w, lay, layers, p, budget_s):
    from block_sparse_gqa_min_b200 import sba
    from block_sparse_gqa_min_b200 import workloads as W

    lay_cpu = W.Layout(lay.seq_lens.cpu(), None if lay.block_table is None else lay.block_table.cpu(),
                       lay.num_pages, lay.max_blocks)

    def fn(l):
        li = layers[l]["li"]
        return W.LayerInputs(li.q.cpu(), li.k.cpu(), li.v.cpu(), li.k_new, li.v_new,
                             None if li.Wq is None else li.Wq.cpu(), None if li.Wk is None else li.Wk.cpu())

    done, t, nbytes = oracle_sample(w, lay_cpu, fn, len(layers), budget_s, lambda N: sba.sba_num_selected(N, p))
    return {"value": round(nbytes / t / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "seconds": round(t, 2), "us_per_step_equiv": round(t / len(done) * len(layers) * 1e6, 1),
            "sample": (f"{len(done)} of {len(layers)} layers (whole layer each: descriptors, scores, selection, "
                       f"fp64 attention), single-threaded C oracle; excludes host copies")}


def reference(args, rank, world):
    """The oracle as the reference arm, on this host's cores."""
    if rank != 0:
        return None
    import numpy as np  # noqa: F401
    import torch

    import oracle as O
    from block_sparse_gqa_min_b200 import workloads as W

    O.build()
    w = W.WORKLOADS[args.workload]
    n_layers = args.layers or w.layers
    lay = W.make_layout(w, args.seed, device="cpu")

    def num_sel(N):
        L = max(w.n_local, 1) if w.scorer == "gate" else w.n_local
        return O.num_selected(N, w.n_budget, L, w.n_min, w.keep_num, w.keep_den)

    cache = {}

    def fn(l):
        if l not in cache:
            cache.clear()
            cache[l] = W.make_layer(w, lay, args.seed, l, device="cpu")
        return cache[l]

    per_step_budget = max(1.0, min(args.cpu_seconds, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, lay, fn, n_layers, 0.0, num_sel)
    times, nbytes_all, layers_all = [], 0, 0
    for _ in range(args.steps):
        done, t, nb = oracle_sample(w, lay, fn, n_layers, per_step_budget, num_sel)
        times.append(t)
        nbytes_all += nb
        layers_all += len(done)
    tot = sum(times)
    value = nbytes_all / tot / 1e9
    ms_step = tot / layers_all * n_layers * 1e3
    torch.set_num_threads(1)
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": {"workload": w.name, "batch": w.B, "layers": n_layers, "H_q": w.H_q, "H_kv": w.H_kv,
                   "block": w.b, "context": [int(lay.seq_lens.min()), int(lay.seq_lens.max())]},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"{layers_all} layer-passes over {args.steps} steps (whole layers, "
                                   f"single-threaded C oracle, fp64)"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        if world > 1:
            import torch.distributed as dist

            dist.init_process_group("gloo")
        out = reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return
    import datetime

    import torch
    import torch.distributed as dist

    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    out = native(args, rank, world, local)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
