"""ctypes binding of ``libseer.so`` -- the names and arguments of include/seer.h.

Argument marshalling only: tensors are passed as raw device pointers and the
stream as its CUDA handle; every step of the computation runs in the CUDA
library. Importing this module loads the library and raises if it has not
been built -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

from . import build as _build

_PKG = os.path.dirname(os.path.abspath(__file__))
HEADER = os.path.join(os.path.dirname(_PKG), "include", "seer.h")

SEER_OK, SEER_ERR_INVALID_ARG, SEER_ERR_UNSUPPORTED, SEER_ERR_CUDA = 0, 1, 2, 3


class SeerError(RuntimeError):
    def __init__(self, fn: str, status: int):
        detail = f" [{LIB.seer_last_error_string().decode()}]" if status == SEER_ERR_CUDA else ""
        super().__init__(f"{fn} failed: {status_string(status)} (status {status}){detail}")
        self.status = status


class seer_dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "num_q_heads", "num_kv_heads", "head_dim", "gate_dim", "block_size", "max_seq_len")]


def _load_library():
    path = _build.LIB
    if not os.path.exists(path):
        raise ImportError(f"libseer.so is not built ({path}); run "
                          "`python -m block_sparse_attention_seer_b200.build` or __graft_entry__.build()")
    lib = ctypes.CDLL(path)
    P, I32, F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    D = ctypes.POINTER(seer_dims)
    sig = {
        "seer_kpool_update": [D, P, P, P, P, P, P],
        "seer_gate_scores": [D, P, P, P, P, P, P],
        "seer_select_blocks": [D, P, P, I32, P, P, P],
        "seer_sparse_decode": [D, P, P, P, P, P, P, I32, I32, F32, P, P, P],
        "seer_combine": [D, P, P, I32, P, P, P],
        "seer_append_kv": [D, P, P, P, P, P, P],
        "seer_block_mass": [D, P, P, P, F32, P, P, P],
        "seer_gate_scores_agg": [D, P, P, P, P, I32, P, P],
        "seer_prefill_gate_scores": [D, P, P, P, P, P, P],
        "seer_prefill_select_blocks": [D, P, P, I32, P, P, P],
        "seer_prefill_attention": [D, P, P, P, P, P, P, I32, F32, P, P, P],
        "seer_select_blocks_threshold": [D, P, P, I32, F32, P, P, P],
        "seer_default_num_splits": [I32, P],
        "seer_decode_wait_failures": [P, I32],
        "seer_decode_step_workspace_size": [D, I32, P],
        "seer_decode_step": [D, P, P, P, P, P, P, P, I32, F32, P, P, P, P, P, P, ctypes.c_size_t, P],
        "seer_decode_step_noalloc": [D, P, P, P, P, P, P, P, I32, F32, P, P, P, P, P, P],
        "seer_wait_selftest": [ctypes.c_int64, P],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.seer_status_string.argtypes = [ctypes.c_int]
    lib.seer_status_string.restype = ctypes.c_char_p
    lib.seer_last_error_string.argtypes = []
    lib.seer_last_error_string.restype = ctypes.c_char_p
    return lib


LIB = _load_library()


def header_functions() -> list[str]:
    """Entry points declared in include/seer.h."""
    text = open(HEADER).read()
    return re.findall(r"^\s*(?:seer_status|const char\*)\s+(seer_\w+)\s*\(", text, flags=re.M)


def status_string(status: int) -> str:
    return LIB.seer_status_string(int(status)).decode()


def make_dims(batch, num_q_heads, num_kv_heads, head_dim, gate_dim, block_size, max_seq_len) -> seer_dims:
    return seer_dims(batch, num_q_heads, num_kv_heads, head_dim, gate_dim, block_size, max_seq_len)


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, torch.Tensor):
        if not x.is_contiguous():
            raise ValueError("tensor arguments must be contiguous")
        return x.data_ptr()
    raise TypeError(f"expected a tensor, int pointer or None, got {type(x)}")


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, status: int):
    if status != SEER_OK:
        raise SeerError(fn, status)


def seer_kpool_update(dims, k_cache, w_k, seq_lens, upd_start, kpool, stream=None):
    _check("seer_kpool_update", LIB.seer_kpool_update(ctypes.byref(dims), _ptr(k_cache), _ptr(w_k), _ptr(seq_lens),
                                                      _ptr(upd_start), _ptr(kpool), _stream(stream)))


def seer_gate_scores(dims, q, w_q, kpool, seq_lens, scores, stream=None):
    _check("seer_gate_scores", LIB.seer_gate_scores(ctypes.byref(dims), _ptr(q), _ptr(w_q), _ptr(kpool),
                                                    _ptr(seq_lens), _ptr(scores), _stream(stream)))


def seer_select_blocks(dims, scores, seq_lens, budget_tokens, block_idx, num_selected, stream=None):
    _check("seer_select_blocks", LIB.seer_select_blocks(ctypes.byref(dims), _ptr(scores), _ptr(seq_lens),
                                                        int(budget_tokens), _ptr(block_idx), _ptr(num_selected),
                                                        _stream(stream)))


def seer_sparse_decode(dims, q, k_cache, v_cache, seq_lens, block_idx, num_selected, kmax, num_splits, sm_scale,
                       o_part, lse_part, stream=None):
    _check("seer_sparse_decode", LIB.seer_sparse_decode(
        ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), _ptr(block_idx),
        _ptr(num_selected), int(kmax), int(num_splits), float(sm_scale), _ptr(o_part), _ptr(lse_part),
        _stream(stream)))


def seer_combine(dims, o_part, lse_part, num_splits, out, lse_out, stream=None):
    _check("seer_combine", LIB.seer_combine(ctypes.byref(dims), _ptr(o_part), _ptr(lse_part), int(num_splits),
                                            _ptr(out), _ptr(lse_out), _stream(stream)))


def seer_prefill_gate_scores(dims, q, w_q, kpool, seq_lens, scores, stream=None):
    """Prefill block scores [B, Hkv, NBmax, NBmax] (query block i, key block j <= i)."""
    _check("seer_prefill_gate_scores", LIB.seer_prefill_gate_scores(ctypes.byref(dims), _ptr(q), _ptr(w_q),
                                                                    _ptr(kpool), _ptr(seq_lens), _ptr(scores),
                                                                    _stream(stream)))


def seer_prefill_select_blocks(dims, scores, seq_lens, budget_tokens, block_idx, num_selected, stream=None):
    """Per query block: itself plus the top min(k, i+1)-1 earlier blocks, ascending."""
    _check("seer_prefill_select_blocks",
           LIB.seer_prefill_select_blocks(ctypes.byref(dims), _ptr(scores), _ptr(seq_lens), int(budget_tokens),
                                          _ptr(block_idx), _ptr(num_selected), _stream(stream)))


def seer_prefill_attention(dims, q, k_cache, v_cache, seq_lens, block_idx, num_selected, kmax, out, lse_out=None,
                           sm_scale=0.0, stream=None):
    """Causal block-sparse attention of every prompt token over its query block's kept blocks."""
    _check("seer_prefill_attention",
           LIB.seer_prefill_attention(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens),
                                      _ptr(block_idx), _ptr(num_selected), int(kmax), float(sm_scale), _ptr(out),
                                      _ptr(lse_out), _stream(stream)))


AGG_MEAN, AGG_MAX, AGG_SOFTMAX_MEAN = 0, 1, 2


def seer_gate_scores_agg(dims, q, w_q, kpool, seq_lens, aggregation, scores, stream=None):
    """Per-head block scores aggregated over the group: AGG_MEAN, AGG_MAX or AGG_SOFTMAX_MEAN."""
    _check("seer_gate_scores_agg", LIB.seer_gate_scores_agg(ctypes.byref(dims), _ptr(q), _ptr(w_q), _ptr(kpool),
                                                            _ptr(seq_lens), int(aggregation), _ptr(scores),
                                                            _stream(stream)))


def seer_select_blocks_threshold(dims, scores, seq_lens, budget_tokens, threshold, block_idx, num_selected,
                                 stream=None):
    """The last block plus at most k_b-1 candidates scoring >= threshold (the highest), ascending."""
    _check("seer_select_blocks_threshold",
           LIB.seer_select_blocks_threshold(ctypes.byref(dims), _ptr(scores), _ptr(seq_lens), int(budget_tokens),
                                            float(threshold), _ptr(block_idx), _ptr(num_selected), _stream(stream)))


def seer_block_mass(dims, q, k_cache, seq_lens, mass, lse_out=None, sm_scale=0.0, stream=None):
    """Each query head's dense softmax mass per KV block -> mass [B, Hq, NBmax], lse [B, Hq]."""
    _check("seer_block_mass", LIB.seer_block_mass(ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(seq_lens),
                                                  float(sm_scale), _ptr(mass), _ptr(lse_out), _stream(stream)))


def seer_append_kv(dims, k_new, v_new, seq_lens, k_cache, v_cache, stream=None):
    """The step's token: K/V rows [B, Hkv, D] -> position L_b - 1 of the caches."""
    _check("seer_append_kv", LIB.seer_append_kv(ctypes.byref(dims), _ptr(k_new), _ptr(v_new), _ptr(seq_lens),
                                                _ptr(k_cache), _ptr(v_cache), _stream(stream)))


def seer_decode_step_workspace_size(dims, budget_tokens) -> int:
    out = ctypes.c_size_t(0)
    _check("seer_decode_step_workspace_size",
           LIB.seer_decode_step_workspace_size(ctypes.byref(dims), int(budget_tokens), ctypes.byref(out)))
    return int(out.value)


def seer_decode_step(dims, q, k_cache, v_cache, w_q, w_k, seq_lens, upd_start, budget_tokens, sm_scale, kpool,
                     block_idx, num_selected, out, lse_out, workspace, workspace_bytes=None, stream=None):
    nbytes = workspace.numel() * workspace.element_size() if workspace_bytes is None else int(workspace_bytes)
    _check("seer_decode_step", LIB.seer_decode_step(
        ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(w_q), _ptr(w_k), _ptr(seq_lens),
        _ptr(upd_start), int(budget_tokens), float(sm_scale), _ptr(kpool), _ptr(block_idx), _ptr(num_selected),
        _ptr(out), _ptr(lse_out), _ptr(workspace), nbytes, _stream(stream)))


def seer_decode_step_noalloc(dims, q, k_cache, v_cache, w_q, w_k, seq_lens, upd_start, budget_tokens, sm_scale,
                             kpool, block_idx, num_selected, out, lse_out, stream=None):
    """seer_decode_step with its scratch in the library's static device array (no workspace, no allocation)."""
    _check("seer_decode_step_noalloc", LIB.seer_decode_step_noalloc(
        ctypes.byref(dims), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(w_q), _ptr(w_k), _ptr(seq_lens),
        _ptr(upd_start), int(budget_tokens), float(sm_scale), _ptr(kpool), _ptr(block_idx), _ptr(num_selected),
        _ptr(out), _ptr(lse_out), _stream(stream)))


def seer_default_num_splits(kmax: int) -> int:
    out = ctypes.c_int32(0)
    _check("seer_default_num_splits", LIB.seer_default_num_splits(int(kmax), ctypes.byref(out)))
    return int(out.value)


def seer_decode_wait_failures(reset: bool = False) -> int:
    out = ctypes.c_uint32(0)
    _check("seer_decode_wait_failures", LIB.seer_decode_wait_failures(ctypes.byref(out), int(bool(reset))))
    return int(out.value)


def seer_wait_selftest(limit_ns: int) -> int:
    out = ctypes.c_int32(-1)
    _check("seer_wait_selftest", LIB.seer_wait_selftest(int(limit_ns), ctypes.byref(out)))
    return int(out.value)


class DecodeStep:
    """Device buffers and the five calls of one decode step for fixed shapes.

    Buffers are allocated once (torch owns them); each call only launches
    kernels on the current stream. Launch count per ``step``: 5.
    """

    def __init__(self, batch, num_q_heads, num_kv_heads, head_dim, gate_dim, block_size, max_seq_len,
                 budget_tokens, device="cuda", num_splits=None):
        self.dims = make_dims(batch, num_q_heads, num_kv_heads, head_dim, gate_dim, block_size, max_seq_len)
        self.budget_tokens = int(budget_tokens)
        self.kmax = self.budget_tokens // block_size
        nb_max = (max_seq_len + block_size - 1) // block_size
        self.nb_max = nb_max
        self.num_splits = int(num_splits) if num_splits else seer_default_num_splits(self.kmax)
        dev = torch.device(device)
        f32, i32 = torch.float32, torch.int32
        self.kpool = torch.zeros(batch, num_kv_heads, nb_max, gate_dim, dtype=f32, device=dev)
        self.scores = torch.zeros(batch, num_kv_heads, nb_max, dtype=f32, device=dev)
        self.block_idx = torch.zeros(batch, num_kv_heads, self.kmax, dtype=i32, device=dev)
        self.num_selected = torch.zeros(batch, num_kv_heads, dtype=i32, device=dev)
        self.out = torch.zeros(batch, num_q_heads, head_dim, dtype=torch.bfloat16, device=dev)
        self.lse = torch.zeros(batch, num_q_heads, dtype=f32, device=dev)
        self.upd_start = torch.zeros(batch, dtype=i32, device=dev)
        self._parts = {}

    def parts(self, num_splits):
        if num_splits not in self._parts:
            d = self.dims
            dev = self.kpool.device
            self._parts[num_splits] = (
                torch.empty(d.batch, d.num_q_heads, num_splits, d.head_dim, dtype=torch.float32, device=dev),
                torch.empty(d.batch, d.num_q_heads, num_splits, dtype=torch.float32, device=dev))
        return self._parts[num_splits]

    def build_pool(self, k_cache, w_k, seq_lens, stream=None):
        """Pooled-K cache of every block (after a prefill)."""
        seer_kpool_update(self.dims, k_cache, w_k, seq_lens, None, self.kpool, stream)

    def set_update_start(self, seq_lens):
        """Decode refresh point: the open last block (start = L_b - 1)."""
        torch.sub(seq_lens, 1, out=self.upd_start)

    def attend(self, q, k_cache, v_cache, seq_lens, block_idx, num_selected, kmax, num_splits=None,
               sm_scale=0.0, stream=None):
        """a4 + a5 on a given block list (e.g. a dense list, or the oracle's)."""
        S = int(num_splits) if num_splits else seer_default_num_splits(kmax)
        o_part, lse_part = self.parts(S)
        seer_sparse_decode(self.dims, q, k_cache, v_cache, seq_lens, block_idx, num_selected, kmax, S, sm_scale,
                           o_part, lse_part, stream)
        seer_combine(self.dims, o_part, lse_part, S, self.out, self.lse, stream)
        return self.out, self.lse

    def workspace(self):
        """Zero-filled scratch of the fused step (allocated once; each call leaves it ready for the next)."""
        if getattr(self, "_ws", None) is None:
            n = seer_decode_step_workspace_size(self.dims, self.budget_tokens)
            self._ws = torch.zeros(n, dtype=torch.uint8, device=self.kpool.device)
        return self._ws

    def fused_step(self, q, k_cache, v_cache, w_q, w_k, seq_lens, sm_scale=0.0, stream=None, upd_start=None):
        """One decode step a1..a5 in a single cooperative launch (seer_decode_step)."""
        seer_decode_step(self.dims, q, k_cache, v_cache, w_q, w_k, seq_lens, upd_start, self.budget_tokens,
                         sm_scale, self.kpool, self.block_idx, self.num_selected, self.out, self.lse,
                         self.workspace(), stream=stream)
        return self.out, self.lse

    def step(self, q, k_cache, v_cache, w_q, w_k, seq_lens, sm_scale=0.0, stream=None):
        """One decode step a1..a5; ``upd_start`` must hold the refresh points (set_update_start)."""
        seer_kpool_update(self.dims, k_cache, w_k, seq_lens, self.upd_start, self.kpool, stream)
        seer_gate_scores(self.dims, q, w_q, self.kpool, seq_lens, self.scores, stream)
        seer_select_blocks(self.dims, self.scores, seq_lens, self.budget_tokens, self.block_idx, self.num_selected,
                           stream)
        return self.attend(q, k_cache, v_cache, seq_lens, self.block_idx, self.num_selected, self.kmax,
                           self.num_splits, sm_scale, stream)

    LAUNCHES_PER_STEP = 5
