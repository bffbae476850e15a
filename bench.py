"""Decode-step benchmark: µs/step and achieved HBM GB/s of the block-sparse GQA
decode path on synthetic workloads shaped like the pages' models.

One step = for every layer: append the step's new K/V tokens, refresh the
descriptors of the touched blocks, score + select, sparse decode, combine --
all through libsba's C ABI, captured once in a CUDA graph and replayed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --sweep [--steps K]     # one line per context, R1-7B and Qwen3-14B shapes
    python bench.py --impl reference ...   # the CPU oracle on a bounded sample

The default workload is the largest single-GPU one, the Qwen3-14B-shaped gated
decode at 524288 tokens (40 layers).  The workload with a rectification window
(R1-7B shape, f = 32) also times the dense rectification pass of all layers and
reports the step with that pass amortised over f steps.

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
DEFAULT_WORKLOAD = "qwen3_14b_gate"
SWEEP_SHAPES = ["r1_7b_256k", "qwen3_14b_gate"]
SWEEP_CONTEXTS = [16384, 32768, 65536, 131072, 262144, 524288]
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
    ap.add_argument("--context", type=int, default=0, help="override the workload's context length")
    ap.add_argument("--sweep", action="store_true",
                    help="one JSON line per context in SWEEP_CONTEXTS for each shape in SWEEP_SHAPES")
    ap.add_argument("--cpu-threads", type=int, default=0, help="threads of the all-cores oracle (0 = affinity)")
    ap.add_argument("--multi", type=int, default=0,
                    help="M > 0: time M query tokens per sequence sharing one selection (Quest workloads)")
    return ap.parse_args()


def select_params_of(w):
    """The C selection rule of a workload (scorer, budget, gate position and activation)."""
    from block_sparse_gqa_min_b200 import sba

    gate = w.scorer == "gate"
    pos = {"off": sba.SBA_LOG_GATE_OFF, "inner": sba.SBA_LOG_GATE_INNER, "outer": sba.SBA_LOG_GATE_OUTER}
    act = {"softmax": sba.SBA_GATE_SOFTMAX, "sigmoid": sba.SBA_GATE_SIGMOID, "raw": sba.SBA_GATE_RAW}
    return sba.select_params(w.n_budget, w.n_local, w.n_min, w.keep_num, w.keep_den,
                             sba.SBA_SCORER_GATE if gate else sba.SBA_SCORER_QUEST,
                             pos[w.gate_position] if gate else 0, act[w.gate_act] if gate else 0)


def workload_of(args):
    from block_sparse_gqa_min_b200 import workloads as W

    w = W.WORKLOADS[args.workload]
    if args.context:
        w = w.with_(len_lo=args.context, len_hi=args.context)
    return w


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


def bf16_peak(sustained: bool = False):
    """Dense bf16 tensor throughput (TFLOP/s) of one B200: the burst figure for a kernel timed
    alone, the sustained one (seconds of back-to-back GEMMs under the power cap) for a kernel
    that runs long enough for the clock to settle."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return float(m["bf16_tflops_sustained" if sustained else "bf16_tflops"]), "measured"
    except Exception:
        return (1400.0 if sustained else 1590.0), "fallback"


# sources of each profiled kernel: a recorded ncu traffic figure is valid only while they are unchanged
KERNEL_SOURCES = {
    "decode_step": ["fused_step.cu", "decode_tile.cuh", "select.cuh", "common.cuh", "launch.cuh"],
    "rectify": ["rect_tc.cu", "common.cuh", "launch.cuh"],
}


def strip_comments(src: str) -> str:
    """C/C++/CUDA source without its comments and blank lines (string and character
    literals kept as they are), so that a comment edit does not count as a kernel change."""
    out, i, n = [], 0, len(src)
    while i < n:
        ch = src[i]
        if ch in "\"'":
            j = i + 1
            while j < n and src[j] != ch:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(ch)
            i += 1
    return "\n".join(line.rstrip() for line in "".join(out).splitlines() if line.strip())


def kernel_source_hash(kernel: str) -> str:
    """Hash of the kernel's sources with comments removed (a recorded ncu traffic figure is
    tied to the code it was measured on)."""
    import hashlib

    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, []):
        with open(os.path.join(ROOT, "block_sparse_gqa_min_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(strip_comments(fh.read()).encode())
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
    if fields.get("source_sha256", "")[:64] != kernel_source_hash(kernel):
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
    p = select_params_of(w)
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


def capture(fn):
    """One CUDA graph of fn() (after one eager run on a side stream)."""
    import torch

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fn()
    torch.cuda.synchronize()
    return graph


def time_graph(graph, steps, warmup, flush_buf, world, local, clocks=True):
    """Mean device time (ms) of one replay over `steps` replays after `warmup`, CUDA events on
    the replay stream; a 512 MB write between replays (outside the events) when flush_buf is
    given.  Returns (ms, clock record)."""
    import torch
    import torch.distributed as dist

    for _ in range(max(warmup, 3)):
        graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local) if clocks else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * steps + 2)]
    if flush_buf is not None:
        for i in range(steps):
            flush_buf.fill_(float(i))
            ev[2 * i].record()
            graph.replay()
            ev[2 * i + 1].record()
        torch.cuda.synchronize()
        total_ms = sum(ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(steps))
    else:
        ev[0].record()
        for _ in range(steps):
            graph.replay()
        ev[1].record()
        torch.cuda.synchronize()
        total_ms = ev[0].elapsed_time(ev[1])
    clk = sampler.stop() if sampler else None
    if world > 1:
        dist.barrier()
    return total_ms / steps, clk


def append_update_bytes(w, lens):
    """Bytes a step writes beyond its counted reads (reported apart, per layer): the appended
    K and V rows, and the refreshed descriptor of every block they touch."""
    tot = 0
    for L in lens:
        p0 = max(int(L) - w.append_tokens, 0)
        touched = (int(L) - 1) // w.b - p0 // w.b + 1 if L > 0 else 0
        tot += w.append_tokens * w.H_kv * w.d * 2 * 2 + touched * w.H_kv * DESC_BYTES
    return tot


def rect_bytes(w, lens):
    """Algorithmic bytes of one rectification pass of one layer: every valid K and V row of the
    cache read once, the window's rows written, the touched blocks' descriptors written."""
    f = w.rectify_every
    tot = 0
    for L in lens:
        L = int(L)
        touched = (L - 1) // w.b - max(L - f, 0) // w.b + 1 if L > 0 else 0
        tot += L * w.H_kv * w.d * 2 * 2 + f * w.H_kv * w.d * 2 * 2 + touched * w.H_kv * DESC_BYTES
    return tot


def rect_flops(w, lens, rows_per_cta=128):
    """Tensor-core work of one rectification pass of one layer: (algorithmic, executed) flops.
    Algorithmic: Q K^T and P V of every query row over the tokens it sees (row i of the window
    sees L - f + i + 1).  Executed: every 64-token stage against every 128-row tile, with P V
    issued twice (P's bf16 hi and lo parts)."""
    f, G, d = w.rectify_every, w.H_q // w.H_kv, w.d
    tiles = -(-f * G // rows_per_cta)
    alg = ex = 0
    for L in lens:
        L = int(L)
        if L <= 0:
            continue
        seen = sum(L - f + i + 1 for i in range(f))
        alg += 4 * d * G * seen * w.H_kv
        ex += 2 * d * rows_per_cta * tiles * (-(-L // 64) * 64) * 3 * w.H_kv
    return alg, ex


def native(args, rank, world, local, w=None, sweep=False):
    import torch

    from block_sparse_gqa_min_b200 import sba
    from block_sparse_gqa_min_b200 import workloads as W

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    sba.load()
    w = w or workload_of(args)
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
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = step_bytes < 4 * l2
    flush_buf = torch.empty((512 * 1024 * 1024 // 4,), dtype=torch.float32, device=dev) if flush else None

    # ---- the rectification pass (every f steps), timed first: the cache it leaves is the one
    # the decode step then runs on, and the one the oracle checks below ----
    rect = None
    if w.rectify_every and args.path == "fused" and not sweep:
        f = w.rectify_every
        rins = [W.make_rect_inputs(w, seed, l, device=dev) for l in range(n_layers)]
        rg = sba.sba_multi_row_groups(layers[0]["c"], f)
        N_max = (lay.max_blocks)
        S_r = max(1, min(N_max, torch.cuda.get_device_properties(dev).multi_processor_count // (w.B * w.H_kv * rg)))
        o_r = torch.empty((w.B, f, w.H_q, S_r, w.d), dtype=torch.float32, device=dev)
        l_r = torch.empty((w.B, f, w.H_q, S_r), dtype=torch.float32, device=dev)
        out_r = torch.empty((w.B, f * w.H_q, w.d), dtype=torch.float32, device=dev)
        lse_r = torch.empty((w.B, f * w.H_q), dtype=torch.float32, device=dev)

        def rect_pass():
            for L, ri in zip(layers, rins):
                sba.sba_rectify(L["c"], ri.q, ri.k_new, ri.v_new, w.scale, o_r, l_r)
                sba.sba_combine(o_r, l_r, out_r, lse_r)

        rgraph = capture(rect_pass)
        r_ms, _ = time_graph(rgraph, max(3, min(args.steps, 10)), args.warmup, None, world, local, clocks=False)
        r_ms = max_over_ranks(r_ms, world, dev)
        rb = rect_bytes(w, lens) * n_layers
        hbm, _ = peaks()
        tc, tc_src = bf16_peak()
        tcs, _ = bf16_peak(sustained=True)
        fa, fe = (x * n_layers for x in rect_flops(w, lens))
        rect = {"every_steps": f, "us_per_pass": round(r_ms * 1e3, 1), "us_per_layer": round(r_ms * 1e3 / n_layers, 2),
                "bytes_per_pass": rb, "gbs": round(job_gbs(rb, world, r_ms), 1),
                "frac_of_measured_hbm": round(job_gbs(rb, 1, r_ms) / hbm, 4),
                "tensor": {"flops_per_pass": fa, "executed_flops_per_pass": fe,
                           "tflops": round(fa / (r_ms * 1e-3) / 1e12, 1),
                           "executed_tflops": round(fe / (r_ms * 1e-3) / 1e12, 1),
                           "peak": tc, "peak_source": tc_src,
                           "frac_executed": round(fe / (r_ms * 1e-3) / 1e12 / tc, 4),
                           "peak_sustained": tcs,
                           "frac_executed_of_sustained": round(fe / (r_ms * 1e-3) / 1e12 / tcs, 4)},
                "num_splits": S_r, "row_groups": rg,
                "kernels": "rect_tc_kernel (tcgen05) + combine_kernel per layer (one CUDA graph)"}
        rt = recorded_traffic("rectify", w.name)
        rect["traffic_per_layer"] = rt
        rect["traffic_over_algorithmic"] = round(rt / (rb / n_layers), 3) if rt else None
        del rgraph

    def step():
        for L in layers:
            layer_step(w, L, p, pos, path=args.path)

    graph = capture(step)
    ms, clk = time_graph(graph, args.steps, args.warmup, flush_buf, world, local)
    ms_max = max_over_ranks(ms, world, dev)
    value = job_gbs(step_bytes, world, ms_max)
    hbm, peak_kind = peaks()
    step_frac = step_bytes / (ms_max * 1e-3) / 1e9 / hbm

    # ---- roofline of the dominant kernel ----
    if args.path == "fused":
        # one launch per layer inside the graph: its in-step duration is the step time over the
        # launches (consecutive layers overlap only by programmatic-dependent-launch prologues)
        launch_ms = ms_max / n_layers
        achieved = per_layer / (launch_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": "decode_step", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "peak_source": peak_kind, "alg_bytes_per_launch": per_layer,
                "launch_us": round(launch_ms * 1e3, 3),
                "launch_us_source": "graph-replayed step time / launches per step (CUDA events)",
                "traffic": recorded_traffic("decode_step", w.name), "step_frac": round(step_frac, 4)}
    else:
        names = ["append_kv", "update_descriptors", "score_select", "sparse_decode", "combine"]
        kt = {k: [] for k in names}
        for _ in range(3):
            torch.cuda._sleep(int(2e8))
            rec = []
            for L in layers:
                c, li, bufs = L["c"], L["li"], L["bufs"]
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
                ev[0].record()
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
        alg = {"sparse_decode": kv_bytes_layer, "score_select": desc_bytes_layer}
        dom = max(alg, key=lambda k: kmean[k])
        achieved = alg[dom] / (kmean[dom] * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "peak_source": peak_kind, "alg_bytes_per_launch": alg[dom],
                "launch_us": round(kmean[dom] * 1e3, 3),
                "launch_us_source": "eager launches behind a sleep kernel (CUDA events)",
                "traffic": recorded_traffic(dom, w.name),
                "other_kernels_us": {k: round(v * 1e3, 3) for k, v in kmean.items() if k != dom},
                "step_frac": round(step_frac, 4)}

    # ---- e2e: host buffers, copies inside the timed region ----
    e2e = None
    if not args.no_e2e and not sweep:
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
            import torch.distributed as dist

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

    # the graph's last replay left the selection of every layer in its buffers (same inputs every
    # replay); the status words must be clean
    graph.replay()
    torch.cuda.synchronize()
    status = [int(L["c"].status.item()) for L in layers]
    if any(status):
        raise RuntimeError(f"device status bits set: {status}")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not sweep:
        cpu = cpu_baseline(w, lay, layers, p, args.cpu_seconds, args.cpu_threads)

    out = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(args.warmup, 3),
        "ms_per_step": round(ms_max, 4),
        "us_per_step": round(ms_max * 1e3, 1),
        "us_per_layer": round(ms_max * 1e3 / n_layers, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; shapes and distributions of the workload, no model weights)",
        "config": {
            "workload": w.name, "batch": w.B, "layers": n_layers, "H_q": w.H_q, "H_kv": w.H_kv, "d": w.d,
            "block": w.b, "context": [min(lens), max(lens)], "blocks_selected_per_group": n_max,
            "scorer": w.scorer, "paged": w.paged, "append_tokens_per_step": w.append_tokens,
            "log_gate": w.gate_position if w.scorer == "gate" else None,
            "gate_act": w.gate_act if w.scorer == "gate" else None,
            "num_splits": splits, "cluster_ctas": sba.sba_decode_step_cluster(layers[0]["c"], p),
            "counted_bytes_per_step": step_bytes,
            "kv_bytes_per_layer": kv_bytes_layer, "desc_bytes_per_layer": desc_bytes_layer,
            "append_update_bytes_per_layer": append_update_bytes(w, lens),
            "l2": (f"L2 flushed between steps (512 MB write, outside the timed events); step footprint "
                   f"{step_bytes / 1e6:.0f} MB" if flush else
                   f"inputs larger than L2: {step_bytes / 1e6:.0f} MB per step vs {l2 / 1e6:.0f} MB L2"),
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
    if rect is not None:
        f = rect["every_steps"]
        amort_ms = ms_max + rect["us_per_pass"] * 1e-3 / f
        rect["step_with_pass_amortised"] = {
            "us_per_step": round(amort_ms * 1e3, 1),
            "gbs": round(job_gbs(step_bytes + rect["bytes_per_pass"] / f, world, amort_ms), 1)}
        out["rectify"] = rect
    del graph
    return out


def native_multi(args, rank, world, local):
    """M query tokens per sequence sharing one selection (sba_score_select_multi +
    sba_sparse_decode_multi + sba_combine per layer, one CUDA graph per step); counted bytes
    as the single-token step (one selection per group reads the same blocks)."""
    import torch

    from block_sparse_gqa_min_b200 import sba
    from block_sparse_gqa_min_b200 import workloads as W

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    sba.load()
    w = workload_of(args)
    if w.scorer != "quest":
        raise SystemExit("--multi: Quest workloads only")
    M = args.multi
    n_layers = args.layers or w.layers
    seed = rank_seed(args.seed, rank)
    lay = W.make_layout(w, seed, device=dev)
    layers, p, pos = build_layers(w, lay, seed, n_layers, dev)
    c0 = layers[0]["c"]
    n_max = layers[0]["bufs"].sel_idx.shape[-1]
    rg = sba.sba_multi_row_groups(c0, M)
    S = max(1, min(n_max, torch.cuda.get_device_properties(dev).multi_processor_count // (w.B * w.H_kv * rg)))
    g = torch.Generator(device=dev)
    g.manual_seed(seed * 7 + M)
    qs = [torch.randn((w.B, M, w.H_q, w.d), generator=g, device=dev).to(torch.bfloat16) for _ in range(n_layers)]
    o_part = torch.empty((w.B, M, w.H_q, S, w.d), dtype=torch.float32, device=dev)
    lse_part = torch.empty((w.B, M, w.H_q, S), dtype=torch.float32, device=dev)
    out = torch.empty((w.B, M * w.H_q, w.d), dtype=torch.float32, device=dev)
    lse = torch.empty((w.B, M * w.H_q), dtype=torch.float32, device=dev)

    def step():
        for L, q in zip(layers, qs):
            b = L["bufs"]
            sba.sba_score_select_multi(L["c"], q, p, b.sel_idx, b.sel_cnt, b.ws)
            sba.sba_sparse_decode_multi(L["c"], q, b.sel_idx, b.sel_cnt, w.scale, o_part, lse_part)
            sba.sba_combine(o_part, lse_part, out, lse)

    graph = capture(step)
    lens = lay.seq_lens.cpu().tolist()
    step_bytes = counted_bytes(w, lens, lambda N: sba.sba_num_selected(N, p)) * n_layers
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = (torch.empty((512 * 1024 * 1024 // 4,), dtype=torch.float32, device=dev)
                 if step_bytes < 4 * l2 else None)
    ms, clk = time_graph(graph, args.steps, args.warmup, flush_buf, world, local)
    ms_max = max_over_ranks(ms, world, dev)
    hbm, peak_kind = peaks()
    gbs = job_gbs(step_bytes, world, ms_max)
    status = [int(L["c"].status.item()) for L in layers]
    if any(status):
        raise RuntimeError(f"device status bits set: {status}")
    del graph
    return {
        "metric": METRIC + f" ({M} query tokens per sequence sharing one selection)",
        "value": round(gbs, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": round(ms_max, 4), "us_per_step": round(ms_max * 1e3, 1),
        "us_per_layer": round(ms_max * 1e3 / n_layers, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded)",
        "config": {"workload": w.name, "query_tokens": M, "batch": w.B, "layers": n_layers, "H_q": w.H_q,
                   "H_kv": w.H_kv, "block": w.b, "context": [min(lens), max(lens)],
                   "blocks_selected_per_group": n_max, "num_splits": S, "row_groups": rg,
                   "counted_bytes_per_step": step_bytes,
                   "graph": "score_select_multi + sparse_decode_multi + combine per layer, one CUDA graph"},
        "roofline": {"bound": "hbm", "kernel": "step", "achieved": round(gbs / world, 1), "peak": hbm,
                     "unit": "GB/s", "frac": round(gbs / world / hbm, 4), "peak_source": peak_kind},
        "gpu_launches": 3 * n_layers * args.steps, "clocks": clk,
    }


# ---------------------------------------------------------------------------
# CPU oracle (timed baseline and the --impl reference arm)
# ---------------------------------------------------------------------------

def _oracle_kwargs(w):
    kw = dict(scale=w.scale, n_budget=w.n_budget, n_local=w.n_local, n_min=w.n_min, keep_num=w.keep_num,
              keep_den=w.keep_den, scorer=w.scorer, log_gate=w.gate_position != "off")
    return kw


def oracle_sample(w, lay_cpu, layer_inputs_fn, n_layers, budget_s, p_num_sel, on_result=None):
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
        kw = _oracle_kwargs(w)
        if w.scorer == "gate":
            kw.update(Wq=li.Wq.cpu().numpy(), Wk=li.Wk.cpu().numpy())
        qb = W.bf16_bits(li.q)
        t0 = time.perf_counter()
        res = O.decode(oc, qb, **kw)
        t_cpu += time.perf_counter() - t0
        if on_result is not None:
            on_result(l, res)
        done.append(l)
        bytes_done += per_layer
        if t_cpu >= budget_s:
            break
    return done, t_cpu, bytes_done


def oracle_all_cores(w, lay_cpu, layer_inputs_fn, n_layers, budget_s, p_num_sel, threads):
    """The same oracle, unchanged, run as independent (layer, sequence, KV group) problems on a
    pool of `threads` threads (the C oracle runs outside the GIL): each problem is the layer's
    cache restricted to one KV head and its G query heads.  Whole layers are taken, in the
    single-threaded sample's order, until about `budget_s` seconds of wall time are used."""
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np

    import oracle as O
    from block_sparse_gqa_min_b200 import workloads as W

    order = sorted(set([0, n_layers - 1, n_layers // 2] + list(range(n_layers))), key=lambda l: (
        0 if l in (0, n_layers - 1, n_layers // 2) else 1, l))
    lens = lay_cpu.seq_lens.tolist()
    per_layer = counted_bytes(w, lens, p_num_sel)
    bt = None if lay_cpu.block_table is None else lay_cpu.block_table.numpy()
    G = w.G
    t_wall, done, nbytes = 0.0, [], 0
    with ThreadPoolExecutor(max_workers=threads) as pool:
        for l in order:
            li = layer_inputs_fn(l)
            kb, vb, qb = W.bf16_bits(li.k), W.bf16_bits(li.v), W.bf16_bits(li.q)
            jobs = []
            for h in range(w.H_kv):  # (the whole batch per head: sequences stay independent inside the oracle)
                oc = O.Cache(np.ascontiguousarray(kb[:, h:h + 1]), np.ascontiguousarray(vb[:, h:h + 1]), bt,
                             lay_cpu.seq_lens.numpy(), H_q=G, max_blocks=lay_cpu.max_blocks)
                kw = _oracle_kwargs(w)
                if w.scorer == "gate":
                    kw.update(Wq=li.Wq.cpu().numpy(), Wk=li.Wk.cpu().numpy())
                jobs.append((oc, np.ascontiguousarray(qb[:, h * G:(h + 1) * G]), kw))
            t0 = time.perf_counter()
            list(pool.map(lambda j: O.decode(j[0], j[1], **j[2]), jobs))
            t_wall += time.perf_counter() - t0
            done.append(l)
            nbytes += per_layer
            if t_wall >= budget_s:
                break
    return done, t_wall, nbytes


def cpu_baseline(w, lay, layers, p, budget_s, threads=0):
    """The oracle timed on this host: all cores (threads over independent KV groups) as the
    reported baseline, single-threaded beside it; the sampled layers' oracle selections are
    compared with the GPU's (exact, near-tie within 1e-5 relative, or mismatch)."""
    import numpy as np

    from block_sparse_gqa_min_b200 import sba
    from block_sparse_gqa_min_b200 import workloads as W

    lay_cpu = W.Layout(lay.seq_lens.cpu(), None if lay.block_table is None else lay.block_table.cpu(),
                       lay.num_pages, lay.max_blocks)
    cache = {}

    def fn(l):
        if l not in cache:
            cache.clear()
            li = layers[l]["li"]
            cache[l] = W.LayerInputs(li.q.cpu(), li.k.cpu(), li.v.cpu(), li.k_new, li.v_new,
                                     None if li.Wq is None else li.Wq.cpu(), None if li.Wk is None else li.Wk.cpu())
        return cache[l]

    sel_check = {"layers": 0, "groups": 0, "exact": 0, "near_tie_events": 0, "mismatch": 0}
    L_eff = max(w.n_local, 1) if w.scorer == "gate" else w.n_local

    def compare(l, ref):
        gi = layers[l]["bufs"].sel_idx.cpu().numpy()
        gc = layers[l]["bufs"].sel_cnt.cpu().numpy()
        sel_check["layers"] += 1
        N_all = ((lay_cpu.seq_lens.numpy().astype(np.int64) + w.b - 1) // w.b)
        for s in range(w.B):
            N = int(N_all[s])
            Lc = min(L_eff, N)
            for h in range(w.H_kv):
                sel_check["groups"] += 1
                n = int(ref.sel_cnt[s, h])
                a, b = set(ref.sel_idx[s, h, :n].tolist()), set(gi[s, h, :int(gc[s, h])].tolist())
                if int(gc[s, h]) == n and a == b:
                    sel_check["exact"] += 1
                    continue
                sc = ref.score[s, h, : N - Lc].astype(np.float32).astype(np.float64)
                adm = [j for j in a if j < N - Lc]
                theta = min(sc[j] for j in adm) if adm else 0.0
                ok = int(gc[s, h]) == n and all(j < N - Lc and abs(sc[j] - theta) <= 1e-5 * abs(theta)
                                                for j in a.symmetric_difference(b))
                sel_check["near_tie_events" if ok else "mismatch"] += 1

    num_sel = lambda N: sba.sba_num_selected(N, p)  # noqa: E731
    done1, t1, nb1 = oracle_sample(w, lay_cpu, fn, len(layers), budget_s, num_sel, on_result=compare)
    threads = threads or len(os.sched_getaffinity(0))
    doneN, tN, nbN = oracle_all_cores(w, lay_cpu, fn, len(layers), budget_s, num_sel, threads)
    return {"value": round(nbN / tN / 1e9, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "seconds": round(tN, 2), "us_per_step_equiv": round(tN / len(doneN) * len(layers) * 1e6, 1),
            "sample": (f"{len(doneN)} of {len(layers)} layers (whole layers: descriptors, scores, selection, fp64 "
                       f"attention), the unchanged C oracle run as independent KV-group problems on {threads} "
                       f"threads; excludes host copies"),
            "single_core": {"value": round(nb1 / t1 / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                            "seconds": round(t1, 2), "us_per_step_equiv": round(t1 / len(done1) * len(layers) * 1e6, 1),
                            "sample": f"{len(done1)} of {len(layers)} whole layers, single-threaded C oracle"},
            "selection_check": sel_check}


def reference(args, rank, world):
    """The oracle as the reference arm, on this host's cores: every step is a bounded sample of
    the workload's layers, run as independent KV-group problems on all the cores this process
    may use.  Every layer of a workload has the same shapes and the same work, so the inputs of
    one layer are generated once (at 512K tokens that alone takes ~30 s of CPU) and the oracle
    re-runs them as each sampled layer."""
    if rank != 0:
        return None
    import torch

    import oracle as O
    from block_sparse_gqa_min_b200 import workloads as W

    O.build()
    w = workload_of(args)
    n_layers = args.layers or w.layers
    lay = W.make_layout(w, args.seed, device="cpu")

    def num_sel(N):
        L = max(w.n_local, 1) if w.scorer == "gate" else w.n_local
        return O.num_selected(N, w.n_budget, L, w.n_min, w.keep_num, w.keep_den)

    li0 = W.make_layer(w, lay, args.seed, 0, device="cpu")

    def fn(l):
        return li0

    threads = args.cpu_threads or len(os.sched_getaffinity(0))
    per_step_budget = max(1.0, min(args.cpu_seconds, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_all_cores(w, lay, fn, n_layers, 0.0, num_sel, threads)
    times, nbytes_all, layers_all = [], 0, 0
    for _ in range(args.steps):
        done, t, nb = oracle_all_cores(w, lay, fn, n_layers, per_step_budget, num_sel, threads)
        times.append(t)
        nbytes_all += nb
        layers_all += len(done)
    tot = sum(times)
    value = nbytes_all / tot / 1e9
    ms_step = tot / layers_all * n_layers * 1e3
    torch.set_num_threads(1)
    lens = lay.seq_lens.tolist()
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3),
        "us_per_step": round(ms_step * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; shapes and distributions of the workload, no model weights)",
        "config": {"workload": w.name, "batch": w.B, "layers": n_layers, "H_q": w.H_q, "H_kv": w.H_kv, "d": w.d,
                   "block": w.b, "context": [min(lens), max(lens)], "scorer": w.scorer, "paged": w.paged},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"{layers_all} layer-passes over {args.steps} steps (whole layers of one "
                                   f"layer's inputs, the unchanged C oracle in fp64 as independent KV-group "
                                   f"problems on {threads} threads)"},
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
    if args.multi:
        out = native_multi(args, rank, world, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
    elif args.sweep:
        # the "vs context" curve: every context at the R1-7B and Qwen3-14B shapes, one line each
        from block_sparse_gqa_min_b200 import workloads as W

        for shape in SWEEP_SHAPES:
            for ctx in SWEEP_CONTEXTS:
                w = W.WORKLOADS[shape].with_(len_lo=ctx, len_hi=ctx)
                out = native(args, rank, world, local, w=w, sweep=True)
                out["config"]["sweep"] = f"{shape} shape at context {ctx}"
                if rank == 0:
                    print(json.dumps(out), flush=True)
                torch.cuda.empty_cache()
    else:
        out = native(args, rank, world, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
