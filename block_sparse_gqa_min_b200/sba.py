"""Thin Python binding of libsba.so (include/sba.h): argument marshalling only.

Every function here has the name of the C entry point it calls and forwards
torch tensors as raw device pointers plus the current CUDA stream.  All
computation happens in the CUDA kernels; there is no CPU path.  If the library
cannot be built or loaded, importing the package raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

from . import _build

SBA_OK = 0
SBA_ERR_INVALID_ARG = 1
SBA_ERR_UNSUPPORTED = 2
SBA_ERR_WORKSPACE = 3
SBA_ERR_CUDA = 4

SBA_DEV_BAD_PAGE = 1
SBA_DEV_BAD_POSITION = 2
SBA_DEV_BAD_SELECTION = 4
SBA_DEV_TIMEOUT = 8

SBA_SCORER_QUEST = 0
SBA_SCORER_GATE = 1
SBA_OUT_F32 = 0
SBA_OUT_BF16 = 1

SBA_LOG_GATE_OFF = 0
SBA_LOG_GATE_INNER = 1
SBA_LOG_GATE_OUTER = 2
SBA_GATE_SOFTMAX = 0
SBA_GATE_SIGMOID = 1
SBA_GATE_RAW = 2


class SbaError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = f"{where}: {sba_status_string(code)} (status {code})"
        if code == SBA_ERR_CUDA:
            msg += f": {load().sba_last_cuda_error().decode()}"
        super().__init__(msg)
        self.code = code


class sba_cache(ctypes.Structure):
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
        ("max_len", ctypes.c_int32),
        ("desc", ctypes.c_void_p),
        ("kg", ctypes.c_void_p),
        ("status", ctypes.c_void_p),
    ]


class sba_gate(ctypes.Structure):
    _fields_ = [("Wq", ctypes.c_void_p), ("Wk", ctypes.c_void_p), ("dg", ctypes.c_int32)]


class sba_select_params(ctypes.Structure):
    _fields_ = [
        ("n_budget", ctypes.c_int32),
        ("n_local", ctypes.c_int32),
        ("n_min", ctypes.c_int32),
        ("keep_num", ctypes.c_int32),
        ("keep_den", ctypes.c_int32),
        ("scorer", ctypes.c_int32),
        ("log_gate", ctypes.c_int32),
        ("gate_act", ctypes.c_int32),
    ]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_SIGS = {
    "sba_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "sba_last_cuda_error": ([], ctypes.c_char_p),
    "sba_num_selected": ([_I, ctypes.POINTER(sba_select_params)], _I),
    "sba_budget_from_sparsity": ([_I, _I, _I], _I),
    "sba_default_num_splits": ([ctypes.POINTER(sba_cache), _I, _I], _I),
    "sba_workspace_size": ([ctypes.POINTER(sba_cache), ctypes.POINTER(sba_select_params)], ctypes.c_size_t),
    "sba_append_kv": ([ctypes.POINTER(sba_cache), _P, _P, _P, _I, _P], ctypes.c_int),
    "sba_update_descriptors": ([ctypes.POINTER(sba_cache), _P, _I, ctypes.POINTER(sba_gate), _P], ctypes.c_int),
    "sba_score_select": ([ctypes.POINTER(sba_cache), _P, ctypes.POINTER(sba_select_params), _P, _P, _P, _I, _P,
                          ctypes.c_size_t, _P], ctypes.c_int),
    "sba_sparse_decode": ([ctypes.POINTER(sba_cache), _P, _P, _P, _P, _I, ctypes.c_float, _I, _P, _P, _P],
                          ctypes.c_int),
    "sba_sparse_decode_outer": ([ctypes.POINTER(sba_cache), _P, _P, _P, _P, _I, ctypes.c_float, _I, _P, _P, _P],
                                ctypes.c_int),
    "sba_score_select_multi": ([ctypes.POINTER(sba_cache), _P, _I, ctypes.POINTER(sba_select_params), _P, _P, _I,
                                _P, ctypes.c_size_t, _P], ctypes.c_int),
    "sba_sparse_decode_multi": ([ctypes.POINTER(sba_cache), _P, _I, _P, _P, _I, ctypes.c_float, _I, _P, _P, _P],
                                ctypes.c_int),
    "sba_multi_row_groups": ([ctypes.POINTER(sba_cache), _I], _I),
    "sba_rectify": ([ctypes.POINTER(sba_cache), _P, _P, _P, _I, ctypes.c_float, _I, _P, _P, _P], ctypes.c_int),
    "sba_combine": ([_P, _P, _I, _I, _I, _I, _P, _I, _P, _P], ctypes.c_int),
    "sba_fold_gate": ([ctypes.POINTER(sba_gate), _P, _P], ctypes.c_int),
    "sba_static_scratch_bytes": ([], ctypes.c_size_t),
    "sba_selftest_wait_timeout": ([_P, ctypes.c_uint64, _P], ctypes.c_int),
    "sba_score_select_static": ([ctypes.POINTER(sba_cache), _P, ctypes.POINTER(sba_select_params), _P, _P, _P, _I,
                                 _P], ctypes.c_int),
    "sba_decode_step_cluster": ([ctypes.POINTER(sba_cache), ctypes.POINTER(sba_select_params)], _I),
    "sba_decode_step": ([ctypes.POINTER(sba_cache), _P, _P, _P, _P, _I, _P, ctypes.POINTER(sba_select_params),
                         ctypes.c_float, _P, _I, _P, _P, _P, _P, _I, _P], ctypes.c_int),
}

_lib = None


def library_path() -> str:
    return _build.LIB


def load() -> ctypes.CDLL:
    """Build libsba.so if it is missing or older than its sources, then load it."""
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        for name, (args, res) in _SIGS.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libsba takes device tensors only")
    if not t.is_contiguous():
        raise ValueError("libsba takes contiguous tensors only")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(rc: int, where: str):
    if rc != SBA_OK:
        raise SbaError(rc, where)


@dataclass
class Cache:
    """Device tensors of one layer's KV cache and its descriptors (sba_cache)."""

    k: torch.Tensor                        # bf16 [num_pages][H_kv][b][d]
    v: torch.Tensor
    seq_lens: torch.Tensor                 # int32 [B]
    H_q: int
    max_blocks: int
    max_len: int
    block_table: Optional[torch.Tensor] = None   # int32 [B][max_blocks]
    desc: Optional[torch.Tensor] = None          # bf16 [num_pages][H_kv][2][d]
    kg: Optional[torch.Tensor] = None            # fp32 [num_pages][H_kv][d]
    status: Optional[torch.Tensor] = None        # int32 [1]

    @property
    def num_pages(self) -> int:
        return int(self.k.shape[0])

    @property
    def H_kv(self) -> int:
        return int(self.k.shape[1])

    @property
    def b(self) -> int:
        return int(self.k.shape[2])

    @property
    def d(self) -> int:
        return int(self.k.shape[3])

    @property
    def B(self) -> int:
        return int(self.seq_lens.shape[0])

    def struct(self) -> sba_cache:
        # rebuilt only when a tensor of the cache is replaced (in-place updates keep the pointers)
        key = (id(self.k), id(self.v), id(self.block_table), id(self.seq_lens), id(self.desc), id(self.kg),
               id(self.status), self.H_q, self.max_blocks, self.max_len)
        cached = self.__dict__.get("_struct")
        if cached is None or cached[0] != key:
            st = sba_cache(_ptr(self.k), _ptr(self.v), _ptr(self.block_table), _ptr(self.seq_lens),
                           self.B, self.H_q, self.H_kv, self.d, self.b, self.max_blocks, self.num_pages,
                           self.max_len, _ptr(self.desc), _ptr(self.kg), _ptr(self.status))
            cached = (key, st)
            self.__dict__["_struct"] = cached
        return cached[1]


def select_params(n_budget=0, n_local=0, n_min=0, keep_num=0, keep_den=0, scorer=SBA_SCORER_QUEST,
                  log_gate=SBA_LOG_GATE_OFF, gate_act=SBA_GATE_SOFTMAX):
    return sba_select_params(n_budget, n_local, n_min, keep_num, keep_den, scorer, log_gate, gate_act)


def sba_status_string(code: int) -> str:
    return load().sba_status_string(code).decode()


def sba_num_selected(N: int, p: sba_select_params) -> int:
    return int(load().sba_num_selected(N, ctypes.byref(p)))


def sba_budget_from_sparsity(N: int, keep_num: int, keep_den: int) -> int:
    return int(load().sba_budget_from_sparsity(N, keep_num, keep_den))


def sba_default_num_splits(c: Cache, n_max: int, num_sms: Optional[int] = None) -> int:
    if num_sms is None:
        num_sms = torch.cuda.get_device_properties(c.k.device).multi_processor_count
    return int(load().sba_default_num_splits(ctypes.byref(c.struct()), n_max, num_sms))


def sba_workspace_size(c: Cache, p: sba_select_params) -> int:
    return int(load().sba_workspace_size(ctypes.byref(c.struct()), ctypes.byref(p)))


def sba_append_kv(c: Cache, k_new: torch.Tensor, v_new: torch.Tensor, pos_start: torch.Tensor, stream=None):
    n_new = int(k_new.shape[1])
    _check(load().sba_append_kv(ctypes.byref(c.struct()), _ptr(k_new), _ptr(v_new), _ptr(pos_start), n_new,
                                _stream(stream)), "sba_append_kv")


def sba_update_descriptors(c: Cache, pos_start: torch.Tensor, n_new: int, Wq: Optional[torch.Tensor] = None,
                           Wk: Optional[torch.Tensor] = None, stream=None):
    gate = None
    if Wq is not None:
        gate = ctypes.byref(sba_gate(_ptr(Wq), _ptr(Wk), int(Wq.shape[0])))
    _check(load().sba_update_descriptors(ctypes.byref(c.struct()), _ptr(pos_start), n_new, gate, _stream(stream)),
           "sba_update_descriptors")


def sba_score_select(c: Cache, q: torch.Tensor, p: sba_select_params, sel_idx: torch.Tensor, sel_cnt: torch.Tensor,
                     gate_bias: Optional[torch.Tensor], ws: torch.Tensor, stream=None):
    n_max = int(sel_idx.shape[-1])
    _check(load().sba_score_select(ctypes.byref(c.struct()), _ptr(q), ctypes.byref(p), _ptr(sel_idx),
                                   _ptr(sel_cnt), _ptr(gate_bias), n_max, _ptr(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)), "sba_score_select")


def sba_static_scratch_bytes() -> int:
    return int(load().sba_static_scratch_bytes())


def sba_score_select_static(c: Cache, q: torch.Tensor, p: sba_select_params, sel_idx: torch.Tensor,
                            sel_cnt: torch.Tensor, gate_bias: Optional[torch.Tensor], stream=None):
    """sba_score_select without a workspace (for callers that cannot allocate):
    the library's static per-device scratch is used instead."""
    n_max = int(sel_idx.shape[-1])
    _check(load().sba_score_select_static(ctypes.byref(c.struct()), _ptr(q), ctypes.byref(p), _ptr(sel_idx),
                                          _ptr(sel_cnt), _ptr(gate_bias), n_max, _stream(stream)),
           "sba_score_select_static")


def sba_sparse_decode(c: Cache, q: torch.Tensor, sel_idx: torch.Tensor, sel_cnt: torch.Tensor,
                      gate_bias: Optional[torch.Tensor], softmax_scale: float, o_part: torch.Tensor,
                      lse_part: torch.Tensor, stream=None):
    n_max = int(sel_idx.shape[-1])
    num_splits = int(lse_part.shape[-1])
    _check(load().sba_sparse_decode(ctypes.byref(c.struct()), _ptr(q), _ptr(sel_idx), _ptr(sel_cnt),
                                    _ptr(gate_bias), n_max, float(softmax_scale), num_splits, _ptr(o_part),
                                    _ptr(lse_part), _stream(stream)), "sba_sparse_decode")


def sba_sparse_decode_outer(c: Cache, q: torch.Tensor, sel_idx: torch.Tensor, sel_cnt: torch.Tensor,
                            gate_bias: torch.Tensor, softmax_scale: float, o_part: torch.Tensor,
                            lse_part: torch.Tensor, stream=None):
    n_max = int(sel_idx.shape[-1])
    num_splits = int(lse_part.shape[-1])
    _check(load().sba_sparse_decode_outer(ctypes.byref(c.struct()), _ptr(q), _ptr(sel_idx), _ptr(sel_cnt),
                                          _ptr(gate_bias), n_max, float(softmax_scale), num_splits, _ptr(o_part),
                                          _ptr(lse_part), _stream(stream)), "sba_sparse_decode_outer")


def sba_score_select_multi(c: Cache, q: torch.Tensor, p: sba_select_params, sel_idx: torch.Tensor,
                           sel_cnt: torch.Tensor, ws: torch.Tensor, stream=None):
    """q: bf16 [B][M][H_q][d]; one Quest selection per (sequence, group) for all M tokens."""
    M = int(q.shape[1])
    n_max = int(sel_idx.shape[-1])
    _check(load().sba_score_select_multi(ctypes.byref(c.struct()), _ptr(q), M, ctypes.byref(p), _ptr(sel_idx),
                                         _ptr(sel_cnt), n_max, _ptr(ws), ws.numel() * ws.element_size(),
                                         _stream(stream)), "sba_score_select_multi")


def sba_multi_row_groups(c: Cache, M: int) -> int:
    return int(load().sba_multi_row_groups(ctypes.byref(c.struct()), M))


def sba_sparse_decode_multi(c: Cache, q: torch.Tensor, sel_idx: torch.Tensor, sel_cnt: torch.Tensor,
                            softmax_scale: float, o_part: torch.Tensor, lse_part: torch.Tensor, stream=None):
    """q: bf16 [B][M][H_q][d]; o_part fp32 [B][M][H_q][S][d], lse_part [B][M][H_q][S]."""
    M = int(q.shape[1])
    n_max = int(sel_idx.shape[-1])
    num_splits = int(lse_part.shape[-1])
    _check(load().sba_sparse_decode_multi(ctypes.byref(c.struct()), _ptr(q), M, _ptr(sel_idx), _ptr(sel_cnt), n_max,
                                          float(softmax_scale), num_splits, _ptr(o_part), _ptr(lse_part),
                                          _stream(stream)), "sba_sparse_decode_multi")


def sba_rectify(c: Cache, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, softmax_scale: float,
                o_part: torch.Tensor, lse_part: torch.Tensor, stream=None):
    """q: bf16 [B][f][H_q][d]; k_new, v_new bf16 [B][f][H_kv][d] (the last f positions)."""
    f = int(q.shape[1])
    num_splits = int(lse_part.shape[-1])
    _check(load().sba_rectify(ctypes.byref(c.struct()), _ptr(q), _ptr(k_new), _ptr(v_new), f, float(softmax_scale),
                              num_splits, _ptr(o_part), _ptr(lse_part), _stream(stream)), "sba_rectify")


def sba_combine(o_part: torch.Tensor, lse_part: torch.Tensor, out: torch.Tensor,
                lse_out: Optional[torch.Tensor] = None, stream=None):
    if o_part.dim() == 5:  # multi-token partials [B][M][H_q][S][d]: merge M*H_q rows
        o_part = o_part.view(o_part.shape[0], -1, o_part.shape[3], o_part.shape[4])
    B, H_q, S, d = o_part.shape
    dt = SBA_OUT_BF16 if out.dtype == torch.bfloat16 else SBA_OUT_F32
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out must be fp32 or bf16")
    _check(load().sba_combine(_ptr(o_part), _ptr(lse_part), B, H_q, S, d, _ptr(out), dt, _ptr(lse_out),
                              _stream(stream)), "sba_combine")


def sba_fold_gate(Wq: torch.Tensor, Wk: torch.Tensor, A: torch.Tensor, stream=None):
    _check(load().sba_fold_gate(ctypes.byref(sba_gate(_ptr(Wq), _ptr(Wk), int(Wq.shape[0]))), _ptr(A),
                                _stream(stream)), "sba_fold_gate")


def sba_selftest_wait_timeout(status: torch.Tensor, limit_ns: int, stream=None):
    """Let one bounded wait run out on purpose (nothing arrives on its barrier): SBA_DEV_TIMEOUT
    is OR-ed into the int32 device `status`, the kernel returns."""
    _check(load().sba_selftest_wait_timeout(_ptr(status), int(limit_ns), _stream(stream)),
           "sba_selftest_wait_timeout")


def sba_decode_step_cluster(c: Cache, p: sba_select_params) -> int:
    return int(load().sba_decode_step_cluster(ctypes.byref(c.struct()), ctypes.byref(p)))


def sba_decode_step(c: Cache, q: torch.Tensor, p: sba_select_params, softmax_scale: float, out: torch.Tensor,
                    lse_out: Optional[torch.Tensor] = None, k_new: Optional[torch.Tensor] = None,
                    v_new: Optional[torch.Tensor] = None, pos_start: Optional[torch.Tensor] = None,
                    gate_A: Optional[torch.Tensor] = None, sel_idx: Optional[torch.Tensor] = None,
                    sel_cnt: Optional[torch.Tensor] = None, gate_bias: Optional[torch.Tensor] = None,
                    stream=None):
    n_new = 0 if k_new is None else int(k_new.shape[1])
    n_max = int(sel_idx.shape[-1]) if sel_idx is not None else (int(gate_bias.shape[-1]) if gate_bias is not None
                                                               else 0)
    dt = SBA_OUT_BF16 if out.dtype == torch.bfloat16 else SBA_OUT_F32
    _check(load().sba_decode_step(ctypes.byref(c.struct()), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(pos_start),
                                  n_new, _ptr(gate_A), ctypes.byref(p), float(softmax_scale), _ptr(out), dt,
                                  _ptr(lse_out), _ptr(sel_idx), _ptr(sel_cnt), _ptr(gate_bias), n_max,
                                  _stream(stream)), "sba_decode_step")


# ---------------------------------------------------------------------------
# Buffers of one decode step (allocation only; every step runs in the kernels)
# ---------------------------------------------------------------------------

@dataclass
class StepBuffers:
    sel_idx: torch.Tensor
    sel_cnt: torch.Tensor
    gate_bias: Optional[torch.Tensor]
    o_part: torch.Tensor
    lse_part: torch.Tensor
    out: torch.Tensor
    lse: torch.Tensor
    ws: torch.Tensor


def alloc_step(c: Cache, p: sba_select_params, num_splits: Optional[int] = None, n_max: Optional[int] = None,
               out_dtype=torch.float32) -> StepBuffers:
    dev = c.k.device
    N_max = (c.max_len + c.b - 1) // c.b
    if n_max is None:
        n_max = max(1, sba_num_selected(N_max, p))
    if num_splits is None:
        num_splits = sba_default_num_splits(c, n_max)
    ws_bytes = sba_workspace_size(c, p)
    return StepBuffers(
        sel_idx=torch.full((c.B, c.H_kv, n_max), -1, dtype=torch.int32, device=dev),
        sel_cnt=torch.zeros((c.B, c.H_kv), dtype=torch.int32, device=dev),
        gate_bias=(torch.zeros((c.B, c.H_q, n_max), dtype=torch.float32, device=dev)
                   if p.scorer == SBA_SCORER_GATE else None),
        o_part=torch.empty((c.B, c.H_q, num_splits, c.d), dtype=torch.float32, device=dev),
        lse_part=torch.empty((c.B, c.H_q, num_splits), dtype=torch.float32, device=dev),
        out=torch.empty((c.B, c.H_q, c.d), dtype=out_dtype, device=dev),
        lse=torch.empty((c.B, c.H_q), dtype=torch.float32, device=dev),
        ws=torch.zeros(((ws_bytes + 15) // 16 * 16,), dtype=torch.uint8, device=dev),
    )


def decode_step(c: Cache, q: torch.Tensor, p: sba_select_params, bufs: StepBuffers, softmax_scale: float,
                stream=None):
    """score_select -> sparse_decode -> combine for one layer (three library calls; the gate's
    position p.log_gate picks the decode call and whether it gets the log-gates)."""
    sba_score_select(c, q, p, bufs.sel_idx, bufs.sel_cnt, bufs.gate_bias, bufs.ws, stream)
    gate = p.scorer == SBA_SCORER_GATE
    if gate and p.log_gate == SBA_LOG_GATE_OUTER:
        sba_sparse_decode_outer(c, q, bufs.sel_idx, bufs.sel_cnt, bufs.gate_bias, softmax_scale, bufs.o_part,
                                bufs.lse_part, stream)
    else:
        bias = bufs.gate_bias if (gate and p.log_gate == SBA_LOG_GATE_INNER) else None
        sba_sparse_decode(c, q, bufs.sel_idx, bufs.sel_cnt, bias, softmax_scale, bufs.o_part, bufs.lse_part, stream)
    sba_combine(bufs.o_part, bufs.lse_part, bufs.out, bufs.lse, stream)
