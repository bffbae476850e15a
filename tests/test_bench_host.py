"""Host-side checks of the measurement plumbing in bench.py (no GPU).

The counted bytes per layer are pinned to the closed form the workloads imply
(selected K and V blocks in bf16 plus one 512-byte descriptor per block and KV
head), worked out by hand for the four model-shaped workloads; the recorded
ncu traffic is used only while the kernel sources match the summary's hash.
"""
from __future__ import annotations

import pytest

import bench
from block_sparse_gqa_min_b200 import sba
from block_sparse_gqa_min_b200 import workloads as W

MiB = 1 << 20


def _params(w: W.Workload):
    return sba.select_params(w.n_budget, w.n_local, w.n_min, w.keep_num, w.keep_den,
                             sba.SBA_SCORER_GATE if w.scorer == "gate" else sba.SBA_SCORER_QUEST)


@pytest.mark.parametrize("name,expect", [
    # 64 blocks x 64 tokens x 128 ch x (K,V) x 2 B x 8 heads + 512 blocks x 8 heads x 512 B
    ("qwen3_4b", 16 * MiB + 2 * MiB),
    # ceil(0.05 x 2048) = 103 blocks x 128 tokens x ... x 4 heads + 2048 x 4 x 512 B
    ("r1_7b_256k", 103 * 128 * 128 * 2 * 2 * 4 + 4 * MiB),
    # 32 blocks x 64 tokens x ... x 8 heads + 8192 x 8 x 512 B
    ("qwen3_14b_gate", 8 * MiB + 32 * MiB),
])
def test_counted_bytes_closed_form(name, expect):
    w = W.WORKLOADS[name]
    p = _params(w)
    got = bench.counted_bytes(w, [w.len_hi] * w.B, lambda N: sba.sba_num_selected(N, p))
    assert got == expect


def test_counted_bytes_paged_sums_sequences():
    """Ragged batch: every sequence counts its own blocks and its own selection."""
    w = W.WORKLOADS["paged_b8"]
    lens = [32768, 32769, 65536]
    per = [(512, 32), (513, 32), (1024, 32)]
    expect = sum(n * 64 * 128 * 4 * 8 + N * 8 * 512 for N, n in per)
    assert bench.counted_bytes(w.with_(B=3), lens, lambda N: 32) == expect


def test_job_throughput_is_all_ranks_over_the_slowest():
    assert bench.job_gbs(10**9, 1, 1000.0) == pytest.approx(1.0)
    assert bench.job_gbs(10**9, 4, 500.0) == pytest.approx(8.0)


def test_recorded_traffic_follows_the_source_hash(monkeypatch):
    w = "qwen3_4b"
    real = bench.kernel_source_hash("decode_step")
    val = bench.recorded_traffic("decode_step", w)
    text = open(f"{bench.ROOT}/profiles/decode_step_{w}.md").read()
    if f"source_sha256: `{real}`" in text:
        assert isinstance(val, int) and val > 0
    else:
        assert val is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kernel: "0" * 64)
    assert bench.recorded_traffic("decode_step", w) is None          # kernel changed since the capture
    assert bench.recorded_traffic("decode_step", "no_such_workload") is None


def test_rectification_counts_closed_form():
    """R1-7B, f = 32, one sequence of 262144 tokens, 4 KV heads of G = 7 query heads:
    bytes = every K and V row read once + the window's rows written + the touched blocks'
    descriptors written; algorithmic flops = 4 d G sum_i (L - f + i + 1) per head (Q K^T and
    P V over the tokens each query row sees); executed = 2 rows-tiles of 128 rows x every
    64-token tile x 128 channels x 2 flops x 3 (S once, P V for P's hi and lo parts)."""
    w = W.WORKLOADS["r1_7b_256k"]
    L, f, d, G, H = 262144, 32, 128, 7, 4
    assert bench.rect_bytes(w, [L]) == L * H * d * 2 * 2 + f * H * d * 2 * 2 + 1 * H * 512
    alg, ex = bench.rect_flops(w, [L])
    seen = f * (L - f) + f * (f + 1) // 2
    assert alg == 4 * d * G * seen * H
    assert ex == 2 * d * 128 * 2 * L * 3 * H     # 224 rows -> two 128-row tiles; L is a multiple of 64
    # a window crossing a block boundary touches two blocks
    assert bench.rect_bytes(w, [L + 16]) - bench.rect_bytes(w, [L]) == 16 * H * d * 2 * 2 + H * 512


def test_source_hash_ignores_comments_only():
    src = 'int a = 1; // one\n/* two */ asm("x; // kept");\n'
    assert bench.strip_comments(src) == bench.strip_comments('int a = 1;\n asm("x; // kept");  // other\n')
    assert bench.strip_comments(src) != bench.strip_comments('int a = 2; // one\n asm("x; // kept");\n')
    assert "// kept" in bench.strip_comments(src)  # string literals are code
