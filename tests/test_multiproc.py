"""Multi-rank host logic of bench.py on CPU with gloo, world size 2: every rank
gets its own batch (distinct seeds, same shapes), the step time is the max over
ranks and the job throughput counts every rank's bytes.  The data path itself
has no collective."""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    from block_sparse_gqa_min_b200 import workloads as W

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.WORKLOADS["paged_b8"].with_(B=2, len_lo=300, len_hi=900, layers=1)
        seed = bench.rank_seed(0, rank)
        lay = W.make_layout(w, seed)
        li = W.make_layer(w, lay, seed, 0)
        ms_local = 1.0 + rank * 0.5           # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms_local, world)
        lens = lay.seq_lens.tolist()
        nbytes = bench.counted_bytes(w, lens, lambda N: min(N, 32))
        total = torch.tensor([nbytes], dtype=torch.float64)
        dist.all_reduce(total)
        out[rank] = dict(seed=seed, lens=lens, q0=float(li.q.float()[0, 0, 0]), ms_max=ms_max,
                         gbs=bench.job_gbs(nbytes, world, ms_max), total=float(total.item()), nbytes=nbytes)
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_host_logic():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    r0, r1 = out[0], out[1]
    assert r0["seed"] != r1["seed"]
    assert r0["q0"] != r1["q0"]                          # independent batches
    assert r0["ms_max"] == r1["ms_max"] == 1.5           # max over ranks, agreed by both
    assert r0["nbytes"] > 0 and r1["nbytes"] > 0
    # job throughput: every rank's bytes (equal-shape batches: world x per-rank) over the max time
    assert r0["gbs"] == pytest.approx(r0["nbytes"] * 2 / 1.5e-3 / 1e9)
    assert r0["total"] == pytest.approx(r0["nbytes"] + r1["nbytes"])
