"""Plain CPU oracle for group-shared block-sparse decode attention.

TEST INFRASTRUCTURE ONLY: the test-suite, the smoke check and the benchmark's
CPU-baseline leg import this package; the product path never does.  The
arithmetic lives in ``sba_oracle.c`` (double precision, plain loops, in the
order the method is stated); this module only marshals numpy arrays into it.
It shares nothing with the CUDA library.

Sources (page title, section): "Rectified Sparse Attention for Efficient
Long-Sequence Generation" (Summary, Key points, References: Quest,
Flash-Decoding, PagedAttention); "SAS: Simple Attention Sparsification via
End-to-End Optimization of Context Ranking" (Method, Limitations);
"SeerAttention-R: Sparse Attention Adaptation for Long Reasoning" (abstract).

Parity status of each function is pinned by tests/test_oracle_pins.py (swept
by tests/test_oracle_properties.py, guarded by tests/test_oracle_mutations.py);
the end-to-end numbers are "parity unpinned" against the pages (they print no
worked example), so correctness rests on those pins.  The modules
``sas_variants`` and ``multi_query`` extend it to the next rows of the build
(pinned by their own test files) and have no CUDA counterpart yet.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sba_oracle.c")
_LIB = os.path.join(_HERE, "_liboracle.so")


def build(force: bool = False) -> str:
    """Compile sba_oracle.c into _liboracle.so with gcc (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


class _Cache(ctypes.Structure):
    _fields_ = [
        ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p),
        ("B", ctypes.c_int32),
        ("H_q", ctypes.c_int32),
        ("H_kv", ctypes.c_int32),
        ("d", ctypes.c_int32),
        ("b", ctypes.c_int32),
        ("max_blocks", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
    ]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        lib.orc_quest_desc.argtypes = [P, P, P]
        lib.orc_gate_desc.argtypes = [P, P, I, P, P]
        lib.orc_quest_scores.argtypes = [P, P, P]
        lib.orc_gate_scores.argtypes = [P, P, P, P, I, P, P]
        lib.orc_num_selected.argtypes = [I, I, I, I, I, I]
        lib.orc_num_selected.restype = I
        lib.orc_select.argtypes = [P, P, I, I, I, I, I, I, I, I, I, I, P, P]
        lib.orc_select.restype = I
        lib.orc_attend.argtypes = [P, P, P, P, I, P, D, P, P]
        lib.orc_combine.argtypes = [P, P, I, I, I, I, P, P]
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _as(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


@dataclass
class Cache:
    """Raw cache buffers as numpy arrays (the same bits the GPU holds).

    k, v: uint16 bf16 bit patterns [num_pages][H_kv][b][d];
    block_table: int32 [B][max_blocks] or None (contiguous pages);
    seq_lens: int32 [B].
    """

    k: np.ndarray
    v: np.ndarray
    block_table: Optional[np.ndarray]
    seq_lens: np.ndarray
    H_q: int
    max_blocks: int

    def __post_init__(self):
        self.k = _as(self.k, np.uint16)
        self.v = _as(self.v, np.uint16)
        self.seq_lens = _as(self.seq_lens, np.int32)
        if self.block_table is not None:
            self.block_table = _as(self.block_table, np.int32)
        self.num_pages, self.H_kv, self.b, self.d = self.k.shape
        self.B = int(self.seq_lens.shape[0])
        self._c = _Cache(
            _ptr(self.k), _ptr(self.v), _ptr(self.block_table), _ptr(self.seq_lens),
            self.B, self.H_q, self.H_kv, self.d, self.b, self.max_blocks, self.num_pages,
        )

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv

    def n_blocks(self) -> np.ndarray:
        return (self.seq_lens.astype(np.int64) + self.b - 1) // self.b


def quest_desc(c: Cache):
    """Per-channel (min, max) of each block's valid keys, [B][max_blocks][H_kv][d] each (NaN where no block)."""
    shape = (c.B, c.max_blocks, c.H_kv, c.d)
    mn = np.full(shape, np.nan)
    mx = np.full(shape, np.nan)
    _load().orc_quest_desc(ctypes.byref(c._c), _ptr(mn), _ptr(mx))
    return mn, mx


def gate_desc(c: Cache, Wk: np.ndarray):
    """Pooled [max||min||avg] (3d) and kg = Wk.pooled (dg) per block, fp64."""
    Wk = _as(Wk, np.float32)
    dg = Wk.shape[0]
    pooled = np.full((c.B, c.max_blocks, c.H_kv, 3 * c.d), np.nan)
    kg = np.full((c.B, c.max_blocks, c.H_kv, dg), np.nan)
    _load().orc_gate_desc(ctypes.byref(c._c), _ptr(Wk), dg, _ptr(pooled), _ptr(kg))
    return pooled, kg


def quest_scores(c: Cache, q: np.ndarray) -> np.ndarray:
    """Quest group scores [B][H_kv][max_blocks] in fp64 (NaN past N)."""
    q = _as(q, np.uint16)
    score = np.full((c.B, c.H_kv, c.max_blocks), np.nan)
    _load().orc_quest_scores(ctypes.byref(c._c), _ptr(q), _ptr(score))
    return score


def gate_scores(c: Cache, q: np.ndarray, Wq: np.ndarray, Wk: np.ndarray):
    """Gate group scores [B][H_kv][max_blocks] and log-gates [B][H_q][max_blocks] in fp64."""
    q = _as(q, np.uint16)
    Wq = _as(Wq, np.float32)
    Wk = _as(Wk, np.float32)
    dg = Wq.shape[0]
    score = np.full((c.B, c.H_kv, c.max_blocks), np.nan)
    logg = np.full((c.B, c.H_q, c.max_blocks), np.nan)
    _load().orc_gate_scores(ctypes.byref(c._c), _ptr(q), _ptr(Wq), _ptr(Wk), dg, _ptr(score), _ptr(logg))
    return score, logg


def num_selected(N: int, n_budget: int, n_local: int, n_min: int, keep_num: int = 0, keep_den: int = 0) -> int:
    return int(_load().orc_num_selected(N, n_budget, n_local, n_min, keep_num, keep_den))


def select(score: np.ndarray, seq_lens: np.ndarray, b: int, n_budget: int, n_local: int, n_min: int,
           keep_num: int = 0, keep_den: int = 0, n_max: Optional[int] = None):
    """Top-n selection with forced local blocks; returns (sel_idx [B][H_kv][n_max], sel_cnt [B][H_kv])."""
    score = _as(score, np.float64)
    seq_lens = _as(seq_lens, np.int32)
    B, H_kv, max_blocks = score.shape
    if n_max is None:
        n_max = max(1, max_blocks)
    sel_idx = np.full((B, H_kv, n_max), -1, dtype=np.int32)
    sel_cnt = np.zeros((B, H_kv), dtype=np.int32)
    rc = _load().orc_select(_ptr(score), _ptr(seq_lens), B, H_kv, b, max_blocks, n_budget, n_local,
                            n_min, keep_num, keep_den, n_max, _ptr(sel_idx), _ptr(sel_cnt))
    if rc != 0:
        raise ValueError("selection larger than n_max")
    return sel_idx, sel_cnt


def attend(c: Cache, q: np.ndarray, sel_idx: np.ndarray, sel_cnt: np.ndarray, scale: float,
           bias: Optional[np.ndarray] = None):
    """fp64 softmax attention over the selected blocks; returns (out [B][H_q][d], lse [B][H_q])."""
    q = _as(q, np.uint16)
    sel_idx = _as(sel_idx, np.int32)
    sel_cnt = _as(sel_cnt, np.int32)
    n_max = sel_idx.shape[-1]
    if bias is not None:
        bias = _as(bias, np.float64)
        assert bias.shape == (c.B, c.H_q, c.max_blocks)
    out = np.zeros((c.B, c.H_q, c.d))
    lse = np.zeros((c.B, c.H_q))
    _load().orc_attend(ctypes.byref(c._c), _ptr(q), _ptr(sel_idx), _ptr(sel_cnt), n_max, _ptr(bias),
                       float(scale), _ptr(out), _ptr(lse))
    return out, lse


def combine(o_part: np.ndarray, lse_part: np.ndarray):
    """LSE merge of split partials o_part [B][H_q][S][d], lse_part [B][H_q][S]."""
    o_part = _as(o_part, np.float64)
    lse_part = _as(lse_part, np.float64)
    B, H_q, S, d = o_part.shape
    out = np.zeros((B, H_q, d))
    lse = np.zeros((B, H_q))
    _load().orc_combine(_ptr(o_part), _ptr(lse_part), B, H_q, S, d, _ptr(out), _ptr(lse))
    return out, lse


@dataclass
class Decoded:
    score: np.ndarray          # fp64 group scores [B][H_kv][max_blocks]
    sel_idx: np.ndarray        # [B][H_kv][n_max]
    sel_cnt: np.ndarray        # [B][H_kv]
    logg: Optional[np.ndarray]  # fp64 log-gates [B][H_q][max_blocks] (gate scorer only)
    out: np.ndarray            # fp64 [B][H_q][d]
    lse: np.ndarray            # fp64 [B][H_q]


def decode(c: Cache, q: np.ndarray, *, scale: float, n_budget: int, n_local: int, n_min: int,
           keep_num: int = 0, keep_den: int = 0, scorer: str = "quest",
           Wq: Optional[np.ndarray] = None, Wk: Optional[np.ndarray] = None,
           log_gate: bool = True, n_max: Optional[int] = None) -> Decoded:
    """Whole decode step: descriptors -> scores -> selection -> attention."""
    if scorer == "quest":
        score = quest_scores(c, q)
        logg = None
        L = n_local
    elif scorer == "gate":
        score, logg = gate_scores(c, q, Wq, Wk)
        L = max(n_local, 1)  # the current block B0 is always kept
    else:
        raise ValueError(scorer)
    if n_max is None:
        n_max = max(1, c.max_blocks)
    sel_idx, sel_cnt = select(score, c.seq_lens, c.b, n_budget, L, n_min, keep_num, keep_den, n_max)
    bias = logg if (scorer == "gate" and log_gate) else None
    out, lse = attend(c, q, sel_idx, sel_cnt, scale, bias)
    return Decoded(score, sel_idx, sel_cnt, logg, out, lse)
