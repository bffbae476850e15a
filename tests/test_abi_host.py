"""C-ABI checks that need no GPU: the library loads, exports every symbol that
include/sba.h declares, its host helpers agree with the oracle, and bad
arguments are rejected on the host before anything is enqueued."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

import oracle as O
from block_sparse_gqa_min_b200 import sba

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "sba.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sba_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol():
    lib = sba.load()
    names = _declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    for code in range(5):
        assert sba.sba_status_string(code)
    assert "unknown" in sba.sba_status_string(99)


@pytest.mark.parametrize("scorer", [0, 1])
def test_num_selected_matches_oracle(scorer):
    for N in range(0, 70):
        for nb in (0, 1, 5, 16, 64):
            for L in (0, 1, 2, 4):
                for nm in (0, 3, 16):
                    p = sba.select_params(nb, L, nm, 0, 0, scorer)
                    Lo = max(L, 1) if scorer == 1 else L
                    assert sba.sba_num_selected(N, p) == O.num_selected(N, nb, Lo, nm), (N, nb, L, nm)
    p = sba.select_params(0, 4, 16, 5, 100, 0)
    for N in (1, 10, 100, 320, 2048, 2049, 8192):
        assert sba.sba_num_selected(N, p) == O.num_selected(N, 0, 4, 16, 5, 100)


def test_budget_from_sparsity():
    assert sba.sba_budget_from_sparsity(2048, 5, 100) == 103
    assert sba.sba_budget_from_sparsity(2000, 5, 100) == 100
    assert sba.sba_budget_from_sparsity(1, 1, 10) == 1
    assert sba.sba_budget_from_sparsity(10, 0, 10) == 0


def _cache(**kw):
    base = dict(k=0x1000, v=0x2000, block_table=None, seq_lens=0x3000, B=1, H_q=8, H_kv=2, d=128, b=64,
                max_blocks=64, num_pages=64, max_len=4096, desc=0x4000, kg=None, status=None)
    base.update(kw)
    return sba.sba_cache(**base)


def _score(c, q=0x5000, sel=0x6000, cnt=0x7000, n_max=16, ws=0x8000, ws_bytes=1 << 20, p=None):
    lib = sba.load()
    p = p or sba.select_params(16, 2, 0, 0, 0, 0)
    return lib.sba_score_select(ctypes.byref(c), q, ctypes.byref(p), sel, cnt, None, n_max, ws, ws_bytes, None)


def test_rejects_bad_cache_arguments_on_host():
    E_ARG, E_UNS = sba.SBA_ERR_INVALID_ARG, sba.SBA_ERR_UNSUPPORTED
    assert _score(_cache(k=None)) == E_ARG
    assert _score(_cache(seq_lens=None)) == E_ARG
    assert _score(_cache(k=0x1001)) == E_ARG            # misaligned
    assert _score(_cache(d=64)) == E_UNS
    assert _score(_cache(b=32)) == E_UNS
    assert _score(_cache(H_q=7)) == E_ARG               # not a multiple of H_kv
    assert _score(_cache(H_q=34, H_kv=2)) == E_UNS      # G = 17 > 16
    assert _score(_cache(max_len=64 * 64 + 1)) == E_ARG
    assert _score(_cache(num_pages=10)) == E_ARG        # contiguous pages need B*max_blocks
    assert _score(_cache(max_blocks=40000, num_pages=40000, max_len=4096)) == E_UNS


def test_rejects_bad_score_select_arguments_on_host():
    c = _cache()
    assert _score(c, q=None) == sba.SBA_ERR_INVALID_ARG
    assert _score(c, n_max=15) == sba.SBA_ERR_INVALID_ARG          # 16 blocks can be selected
    assert _score(c, ws=None) == sba.SBA_ERR_WORKSPACE
    assert _score(c, ws_bytes=16) == sba.SBA_ERR_WORKSPACE
    assert _score(_cache(desc=None)) == sba.SBA_ERR_INVALID_ARG    # Quest needs descriptors
    gate = sba.select_params(16, 2, 0, 0, 0, 1)
    assert _score(c, p=gate) == sba.SBA_ERR_INVALID_ARG            # gate needs kg
    bad = sba.select_params(16, 2, 0, 5, 4, 0)                      # keep fraction > 1
    assert _score(c, p=bad) == sba.SBA_ERR_INVALID_ARG


def test_workspace_size_is_deterministic_and_covers_scores():
    lib = sba.load()
    c = _cache()
    p = sba.select_params(16, 2, 0, 0, 0, 0)
    n = lib.sba_workspace_size(ctypes.byref(c), ctypes.byref(p))
    assert n >= 4 * 1 * 2 * 64 and n % 256 == 0
    assert n == lib.sba_workspace_size(ctypes.byref(c), ctypes.byref(p))
    pg = sba.select_params(16, 2, 0, 0, 0, 1)
    assert lib.sba_workspace_size(ctypes.byref(_cache(kg=0x9000)), ctypes.byref(pg)) > n
    assert lib.sba_workspace_size(ctypes.byref(_cache(d=64)), ctypes.byref(p)) == 0


def test_rejects_bad_decode_combine_append_update_on_host():
    lib = sba.load()
    c = _cache()
    E = sba.SBA_ERR_INVALID_ARG
    dec = lib.sba_sparse_decode
    assert dec(ctypes.byref(c), 0x5000, 0x6000, 0x7000, None, 16, 0.088, 0, 0x9000, 0xa000, None) == E
    assert dec(ctypes.byref(c), 0x5000, 0x6000, 0x7000, None, 16, -1.0, 4, 0x9000, 0xa000, None) == E
    assert dec(ctypes.byref(c), None, 0x6000, 0x7000, None, 16, 0.088, 4, 0x9000, 0xa000, None) == E
    comb = lib.sba_combine
    assert comb(0x1000, 0x2000, 1, 8, 4, 64, 0x3000, 0, None, None) == sba.SBA_ERR_UNSUPPORTED
    assert comb(0x1000, 0x2000, 1, 8, 4, 128, 0x3000, 7, None, None) == E
    assert comb(None, 0x2000, 1, 8, 4, 128, 0x3000, 0, None, None) == E
    app = lib.sba_append_kv
    assert app(ctypes.byref(c), None, 0x2000, 0x3000, 1, None) == E
    assert app(ctypes.byref(c), 0x1000, 0x2000, 0x3000, 0, None) == sba.SBA_OK   # nothing to do
    upd = lib.sba_update_descriptors
    assert upd(ctypes.byref(c), None, 1, None, None) == E
    g = sba.sba_gate(None, 0x100, 128)
    assert upd(ctypes.byref(c), 0x3000, 1, ctypes.byref(g), None) == E
    assert upd(ctypes.byref(_cache(desc=None)), 0x3000, 1, None, None) == E


def _step(c, q=0x5000, k_new=None, v_new=None, pos=None, n_new=0, gate_A=None, p=None, scale=0.088,
          out=0x9000, out_dtype=0, lse=None, sel=None, cnt=None, gb=None, n_max=0):
    lib = sba.load()
    p = p or sba.select_params(16, 2, 0, 0, 0, 0)
    return lib.sba_decode_step(ctypes.byref(c), q, k_new, v_new, pos, n_new, gate_A, ctypes.byref(p), scale, out,
                               out_dtype, lse, sel, cnt, gb, n_max, None)


def test_rejects_bad_decode_step_arguments_on_host():
    """The fused step checks its arguments before any device work."""
    E = sba.SBA_ERR_INVALID_ARG
    c = _cache()
    assert _step(_cache(k=None)) == E
    assert _step(_cache(d=64)) == sba.SBA_ERR_UNSUPPORTED
    assert _step(c, q=None) == E
    assert _step(c, q=0x5008) == E                      # q not 16-byte aligned
    assert _step(c, out=None) == E
    assert _step(c, out_dtype=7) == E
    assert _step(c, scale=0.0) == E
    assert _step(c, scale=float("nan")) == E
    assert _step(c, scale=float("inf")) == E
    assert _step(c, n_new=-1) == E
    assert _step(c, n_new=1, k_new=0x1000, v_new=0x2000) == E                 # no positions
    assert _step(c, n_new=1, k_new=None, v_new=0x2000, pos=0x3000) == E
    assert _step(c, n_new=1, k_new=0x1008, v_new=0x2000, pos=0x3000) == E     # misaligned rows
    assert _step(_cache(desc=None)) == E                                      # Quest needs descriptors
    gate = sba.select_params(16, 2, 0, 0, 0, 1)
    assert _step(_cache(kg=0x9000), p=gate) == E                              # gate needs the folded A
    assert _step(c, p=gate, gate_A=0xa000) == E                               # ... and stored gate keys
    assert _step(c, sel=0xb000, cnt=0xc000, n_max=15) == E                    # 16 blocks can be selected
    assert _step(c, p=sba.select_params(16, 2, 0, 5, 4, 0)) == E              # keep fraction > 1


def test_rejects_bad_fold_gate_arguments_on_host():
    lib = sba.load()
    E = sba.SBA_ERR_INVALID_ARG
    assert lib.sba_fold_gate(None, 0x1000, None) == E
    for g in (sba.sba_gate(None, 0x100, 128), sba.sba_gate(0x100, None, 128), sba.sba_gate(0x100, 0x200, 0),
              sba.sba_gate(0x100, 0x200, 257)):
        assert lib.sba_fold_gate(ctypes.byref(g), 0x1000, None) == E
    assert lib.sba_fold_gate(ctypes.byref(sba.sba_gate(0x100, 0x200, 128)), None, None) == E


def test_rejects_bad_gate_variant_fields_on_host():
    """log_gate and gate_act take their documented values, and are 0 for the Quest scorer."""
    E = sba.SBA_ERR_INVALID_ARG
    c = _cache(kg=0x9000)
    assert _step(c, p=sba.select_params(16, 2, 0, 0, 0, 1, 3, 0), gate_A=0xa000) == E
    assert _step(c, p=sba.select_params(16, 2, 0, 0, 0, 1, 1, 3), gate_A=0xa000) == E
    assert _step(c, p=sba.select_params(16, 2, 0, 0, 0, 1, -1, 0), gate_A=0xa000) == E
    assert _step(_cache(), p=sba.select_params(16, 2, 0, 0, 0, 0, 1, 0)) == E   # Quest has no log-gate
    assert _step(_cache(), p=sba.select_params(16, 2, 0, 0, 0, 0, 0, 2)) == E


def test_rejects_bad_multi_token_arguments_on_host():
    lib = sba.load()
    E = sba.SBA_ERR_INVALID_ARG
    c = _cache()
    p = sba.select_params(16, 2, 0, 0, 0, 0)
    ssm = lib.sba_score_select_multi
    ws = 0x100000
    assert ssm(ctypes.byref(c), 0x5000, 0, ctypes.byref(p), 0x6000, 0x7000, 16, ws, 1 << 30, None) == E   # M = 0
    assert ssm(ctypes.byref(c), 0x5000, 1025, ctypes.byref(p), 0x6000, 0x7000, 16, ws, 1 << 30, None) == E
    assert ssm(ctypes.byref(c), 0x5008, 4, ctypes.byref(p), 0x6000, 0x7000, 16, ws, 1 << 30, None) == E
    assert ssm(ctypes.byref(c), 0x5000, 4, ctypes.byref(p), 0x6000, 0x7000, 16, None, 0, None) == \
        sba.SBA_ERR_WORKSPACE
    gate = sba.select_params(16, 2, 0, 0, 0, 1, 1, 0)
    assert ssm(ctypes.byref(_cache(kg=0x9000)), 0x5000, 4, ctypes.byref(gate), 0x6000, 0x7000, 16, ws, 1 << 30,
               None) == sba.SBA_ERR_UNSUPPORTED                                    # Quest only
    sdm = lib.sba_sparse_decode_multi
    assert sdm(ctypes.byref(c), 0x5000, 0, 0x6000, 0x7000, 16, 0.088, 2, 0x8000, 0x9000, None) == E
    assert sdm(ctypes.byref(c), 0x5000, 4, None, 0x7000, 16, 0.088, 2, 0x8000, 0x9000, None) == E
    assert sdm(ctypes.byref(c), 0x5000, 4, 0x6000, 0x7000, 16, 0.0, 2, 0x8000, 0x9000, None) == E
    assert sdm(ctypes.byref(c), 0x5000, 4, 0x6000, 0x7000, 16, float("inf"), 2, 0x8000, 0x9000, None) == E
    assert sdm(ctypes.byref(c), 0x5000, 4, 0x6000, 0x7000, 16, 0.088, 0, 0x8000, 0x9000, None) == E
    rect = lib.sba_rectify
    assert rect(ctypes.byref(c), 0x5000, 0x1000, 0x2000, 0, 0.088, 2, 0x8000, 0x9000, None) == E
    assert rect(ctypes.byref(c), 0x5000, 0x1000, 0x2000, 129, 0.088, 2, 0x8000, 0x9000, None) == \
        sba.SBA_ERR_UNSUPPORTED                                                    # window beyond f = 128
    assert rect(ctypes.byref(c), 0x5000, None, 0x2000, 32, 0.088, 2, 0x8000, 0x9000, None) == E
    assert rect(ctypes.byref(c), 0x5000, 0x1000, 0x2000, 32, float("inf"), 2, 0x8000, 0x9000, None) == E
    assert rect(ctypes.byref(c), 0x5000, 0x1008, 0x2000, 32, 0.088, 2, 0x8000, 0x9000, None) == E
    assert lib.sba_multi_row_groups(ctypes.byref(c), 32) == (32 * c.H_q // c.H_kv + 127) // 128
    outer = lib.sba_sparse_decode_outer
    assert outer(ctypes.byref(c), 0x5000, 0x6000, 0x7000, None, 16, 0.088, 2, 0x8000, 0x9000, None) == E  # needs g


def test_rejects_bad_selftest_arguments_on_host():
    lib = sba.load()
    E = sba.SBA_ERR_INVALID_ARG
    assert lib.sba_selftest_wait_timeout(None, 1000, None) == E
    assert lib.sba_selftest_wait_timeout(0x1000, 0, None) == E
    assert lib.sba_selftest_wait_timeout(0x1000, 10_000_000_001, None) == E
