"""Failure detection without a GPU fault: a bounded wait that runs out reports
SBA_DEV_TIMEOUT in the status word, the kernel returns and the CUDA context
stays usable (the next library call computes the right result)."""
from __future__ import annotations

import time

import pytest
import torch

from block_sparse_gqa_min_b200 import sba

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_bounded_wait_runs_out_and_reports():
    dev = torch.device("cuda")
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    sba.sba_selftest_wait_timeout(status, 50_000_000)  # 50 ms
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(status.item()) & sba.SBA_DEV_TIMEOUT
    assert 0.045 <= elapsed < 5.0, elapsed
    # the status bits are OR-ed in: other bits stay
    status.fill_(sba.SBA_DEV_BAD_PAGE)
    sba.sba_selftest_wait_timeout(status, 1_000_000)
    torch.cuda.synchronize()
    assert int(status.item()) == sba.SBA_DEV_BAD_PAGE | sba.SBA_DEV_TIMEOUT


def test_context_usable_after_a_wait_ran_out():
    """After the timeout, a whole step of the tiny workload still matches the oracle."""
    from block_sparse_gqa_min_b200 import workloads as W
    from tests.test_parity_gpu import run_case
    dev = torch.device("cuda")
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    sba.sba_selftest_wait_timeout(status, 10_000_000)
    torch.cuda.synchronize()
    assert int(status.item()) & sba.SBA_DEV_TIMEOUT
    run_case(W.WORKLOADS["tiny"], 0)  # asserts parity and a clean status word itself
