"""Python front of the fp64 CPU oracle (``seer_oracle.c``).

TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's
CPU-baseline leg may import this module. It shares no code with the CUDA
library and never imports it; arrays come in as numpy arrays (bf16 tensors as
their raw ``uint16`` bit patterns) and results go out as float64 / int32 numpy
arrays.

Every function states the step of the method it computes; the C file holds the
arithmetic and cites the pages:
  * "SeerAttention-R: Sparse Attention Adaptation for Long Reasoning" (abstract)
  * "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs" (abstract)
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "seer_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libseer_oracle.so")
_lib = None


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "num_q_heads", "num_kv_heads", "head_dim", "gate_dim", "block_size", "max_seq_len")]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math) into this folder."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall",
                        "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        # SEER_ORACLE_LIB points the pins at another build of the oracle (the
        # mutation test uses it to plant mistakes in a copy of the C file).
        path = os.environ.get("SEER_ORACLE_LIB") or build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_pool_project.argtypes = [ctypes.POINTER(_Dims), P, P, P, P]
        lib.oracle_gate_scores.argtypes = [ctypes.POINTER(_Dims), P, P, P, P, P]
        lib.oracle_select.argtypes = [ctypes.POINTER(_Dims), P, P, ctypes.c_int32, P, P]
        lib.oracle_attend.argtypes = [ctypes.POINTER(_Dims), P, P, P, P, P, P, ctypes.c_int32,
                                      ctypes.c_double, P, P]
        lib.oracle_merge.argtypes = [ctypes.c_int32, ctypes.c_int32, P, P, P, P]
        lib.oracle_block_mass.argtypes = [ctypes.POINTER(_Dims), P, P, P, ctypes.c_double, P, P]
        lib.oracle_gate_scores_agg.argtypes = [ctypes.POINTER(_Dims), P, P, P, P, ctypes.c_int32, P]
        lib.oracle_select_threshold.argtypes = [ctypes.POINTER(_Dims), P, P, ctypes.c_int32, ctypes.c_double, P, P]
        lib.oracle_prefill_gate.argtypes = [ctypes.POINTER(_Dims), P, P, P, P, P]
        lib.oracle_prefill_select.argtypes = [ctypes.POINTER(_Dims), P, P, ctypes.c_int32, P, P]
        lib.oracle_prefill_attend.argtypes = [ctypes.POINTER(_Dims), P, P, P, P, P, P, ctypes.c_int32,
                                              ctypes.c_double, P, P]
        for f in ("oracle_pool_project", "oracle_gate_scores", "oracle_select", "oracle_attend",
                  "oracle_merge", "oracle_block_mass", "oracle_gate_scores_agg", "oracle_select_threshold",
                  "oracle_prefill_gate", "oracle_prefill_select", "oracle_prefill_attend"):
            getattr(lib, f).restype = None
        _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle runs on (its loops are over (batch, KV head) rows)."""
    return int(_load().oracle_num_threads())


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _dims(B, Hq, Hkv, D, dg, blk, Lmax):
    return _Dims(int(B), int(Hq), int(Hkv), int(D), int(dg), int(blk), int(Lmax))


def num_blocks(length: int, blk: int) -> int:
    return (int(length) + blk - 1) // blk


def pool_project(k_bits, w_k, seq_lens, block_size, gate_dim=None):
    """Pooled-and-projected K of every block (mean pool, then W_k).

    k_bits: uint16 [B, Hkv, Lmax, D] (bf16 bits); w_k: float32 [Hkv, dg, D];
    seq_lens: int32 [B]. Returns float64 [B, Hkv, NBmax, dg]; NaN past NB_b.
    """
    k_bits, kp_ = _c(k_bits, np.uint16)
    B, Hkv, Lmax, D = k_bits.shape
    w_k, wp = _c(w_k, np.float32)
    dg = w_k.shape[1]
    sl, slp = _c(seq_lens, np.int32)
    NBmax = num_blocks(Lmax, block_size)
    out = np.empty((B, Hkv, NBmax, dg), np.float64)
    dm = _dims(B, Hkv, Hkv, D, dg, block_size, Lmax)
    _load().oracle_pool_project(ctypes.byref(dm), kp_, wp, slp, out.ctypes.data_as(ctypes.c_void_p))
    return out


def gate_scores(q_bits, w_q, kpool, seq_lens, block_size, max_seq_len):
    """Block scores s[b, kvh, j] from the un-pooled query and the pooled-K rows.

    q_bits: uint16 [B, Hq, D]; w_q: float32 [Hkv, dg, D]; kpool: float64
    [B, Hkv, NBmax, dg]. Returns float64 [B, Hkv, NBmax]; NaN past NB_b.
    """
    q_bits, qp = _c(q_bits, np.uint16)
    B, Hq, D = q_bits.shape
    w_q, wp = _c(w_q, np.float32)
    Hkv, dg = w_q.shape[0], w_q.shape[1]
    kpool, kpp = _c(kpool, np.float64)
    sl, slp = _c(seq_lens, np.int32)
    NBmax = num_blocks(max_seq_len, block_size)
    assert kpool.shape == (B, Hkv, NBmax, dg)
    out = np.empty((B, Hkv, NBmax), np.float64)
    dm = _dims(B, Hq, Hkv, D, dg, block_size, max_seq_len)
    _load().oracle_gate_scores(ctypes.byref(dm), qp, wp, kpp, slp, out.ctypes.data_as(ctypes.c_void_p))
    return out


def select_blocks(scores, seq_lens, block_size, max_seq_len, budget_tokens):
    """Kept blocks: the last block plus the top k_b-1 others (ties: lower index).

    Returns (block_idx int32 [B, Hkv, kmax] ascending, -1 padded;
    num_selected int32 [B, Hkv]) with kmax = budget_tokens // block_size.
    """
    scores, sp = _c(scores, np.float64)
    B, Hkv, NBmax = scores.shape
    assert NBmax == num_blocks(max_seq_len, block_size)
    sl, slp = _c(seq_lens, np.int32)
    kmax = int(budget_tokens) // block_size
    idx = np.empty((B, Hkv, kmax), np.int32)
    nsel = np.empty((B, Hkv), np.int32)
    dm = _dims(B, Hkv, Hkv, 0, 0, block_size, max_seq_len)
    _load().oracle_select(ctypes.byref(dm), sp, slp, int(budget_tokens),
                          idx.ctypes.data_as(ctypes.c_void_p), nsel.ctypes.data_as(ctypes.c_void_p))
    return idx, nsel


AGG_MEAN, AGG_MAX, AGG_SOFTMAX_MEAN = 0, 1, 2


def gate_scores_agg(q_bits, w_q, kpool, seq_lens, block_size, max_seq_len, aggregation):
    """Block scores with every head scored on its own, then aggregated over the group:
    0 mean, 1 max, 2 mean of each head's softmax over its row's blocks. NaN past NB_b."""
    q_bits, qp = _c(q_bits, np.uint16)
    B, Hq, D = q_bits.shape
    w_q, wp = _c(w_q, np.float32)
    Hkv, dg = w_q.shape[0], w_q.shape[1]
    kpool, kpp = _c(kpool, np.float64)
    sl, slp = _c(seq_lens, np.int32)
    NBmax = num_blocks(max_seq_len, block_size)
    assert kpool.shape == (B, Hkv, NBmax, dg)
    out = np.empty((B, Hkv, NBmax), np.float64)
    dm = _dims(B, Hq, Hkv, D, dg, block_size, max_seq_len)
    _load().oracle_gate_scores_agg(ctypes.byref(dm), qp, wp, kpp, slp, int(aggregation),
                                   out.ctypes.data_as(ctypes.c_void_p))
    return out


def select_threshold(scores, seq_lens, block_size, max_seq_len, budget_tokens, threshold):
    """The last block plus the candidates scoring >= threshold, at most k_b-1 (the highest)."""
    scores, sp = _c(scores, np.float64)
    B, Hkv, NBmax = scores.shape
    assert NBmax == num_blocks(max_seq_len, block_size)
    sl, slp = _c(seq_lens, np.int32)
    kmax = int(budget_tokens) // block_size
    idx = np.empty((B, Hkv, kmax), np.int32)
    nsel = np.empty((B, Hkv), np.int32)
    dm = _dims(B, Hkv, Hkv, 0, 0, block_size, max_seq_len)
    _load().oracle_select_threshold(ctypes.byref(dm), sp, slp, int(budget_tokens), float(threshold),
                                    idx.ctypes.data_as(ctypes.c_void_p), nsel.ctypes.data_as(ctypes.c_void_p))
    return idx, nsel


def prefill_gate(q_bits, w_q, kpool, seq_lens, block_size):
    """Prefill block scores s[b, kvh, i, j] (query block i, key block j <= i); NaN elsewhere.

    q_bits uint16 [B, Hq, Lmax, D]; w_q float32 [Hkv, dg, D]; kpool float64 [B, Hkv, NBmax, dg].
    """
    q_bits, qp = _c(q_bits, np.uint16)
    B, Hq, Lmax, D = q_bits.shape
    w_q, wp = _c(w_q, np.float32)
    Hkv, dg = w_q.shape[0], w_q.shape[1]
    kpool, kpp = _c(kpool, np.float64)
    sl, slp = _c(seq_lens, np.int32)
    nbm = num_blocks(Lmax, block_size)
    out = np.empty((B, Hkv, nbm, nbm), np.float64)
    dm = _dims(B, Hq, Hkv, D, dg, block_size, Lmax)
    _load().oracle_prefill_gate(ctypes.byref(dm), qp, wp, kpp, slp, out.ctypes.data_as(ctypes.c_void_p))
    return out


def prefill_select(scores, seq_lens, block_size, max_seq_len, budget_tokens):
    """Per query block i: block i plus the top min(k, i+1)-1 of blocks < i, ascending.

    Returns (block_idx int32 [B, Hkv, NBmax, kmax] -1 padded, num_selected int32 [B, Hkv, NBmax]).
    """
    scores, sp = _c(scores, np.float64)
    B, Hkv, nbm, _ = scores.shape
    sl, slp = _c(seq_lens, np.int32)
    kmax = int(budget_tokens) // block_size
    idx = np.empty((B, Hkv, nbm, kmax), np.int32)
    nsel = np.empty((B, Hkv, nbm), np.int32)
    dm = _dims(B, Hkv, Hkv, 0, 0, block_size, max_seq_len)
    _load().oracle_prefill_select(ctypes.byref(dm), sp, slp, int(budget_tokens), idx.ctypes.data_as(ctypes.c_void_p),
                                  nsel.ctypes.data_as(ctypes.c_void_p))
    return idx, nsel


def prefill_attend(q_bits, k_bits, v_bits, seq_lens, block_idx, num_selected, block_size, sm_scale=0.0):
    """Causal attention of every prompt token over the kept blocks of its query block.

    q_bits uint16 [B, Hq, Lmax, D]; k/v uint16 [B, Hkv, Lmax, D]; block_idx [B, Hkv, NBmax, kmax].
    Returns (out float64 [B, Hq, Lmax, D], lse float64 [B, Hq, Lmax]); rows past L_b are 0 / -inf.
    """
    q_bits, qp = _c(q_bits, np.uint16)
    k_bits, kp_ = _c(k_bits, np.uint16)
    v_bits, vp = _c(v_bits, np.uint16)
    B, Hq, Lmax, D = q_bits.shape
    Hkv = k_bits.shape[1]
    sl, slp = _c(seq_lens, np.int32)
    block_idx, ip = _c(block_idx, np.int32)
    num_selected, np_ = _c(num_selected, np.int32)
    kmax = block_idx.shape[-1]
    out = np.empty((B, Hq, Lmax, D), np.float64)
    lse = np.empty((B, Hq, Lmax), np.float64)
    dm = _dims(B, Hq, Hkv, D, 0, block_size, Lmax)
    _load().oracle_prefill_attend(ctypes.byref(dm), qp, kp_, vp, slp, ip, np_, int(kmax), float(sm_scale),
                                  out.ctypes.data_as(ctypes.c_void_p), lse.ctypes.data_as(ctypes.c_void_p))
    return out, lse


def attend(q_bits, k_bits, v_bits, seq_lens, block_idx, num_selected, block_size, sm_scale=0.0):
    """Softmax attention of each query head over the valid tokens of its kept blocks.

    q_bits uint16 [B, Hq, D]; k_bits/v_bits uint16 [B, Hkv, Lmax, D];
    block_idx int32 [B, Hkv, kmax]; num_selected int32 [B, Hkv].
    Returns (out float64 [B, Hq, D], lse float64 [B, Hq]).
    """
    q_bits, qp = _c(q_bits, np.uint16)
    k_bits, kp_ = _c(k_bits, np.uint16)
    v_bits, vp = _c(v_bits, np.uint16)
    B, Hq, D = q_bits.shape
    _, Hkv, Lmax, _ = k_bits.shape
    assert v_bits.shape == k_bits.shape
    sl, slp = _c(seq_lens, np.int32)
    block_idx, ip = _c(block_idx, np.int32)
    num_selected, np_ = _c(num_selected, np.int32)
    kmax = block_idx.shape[-1]
    out = np.empty((B, Hq, D), np.float64)
    lse = np.empty((B, Hq), np.float64)
    dm = _dims(B, Hq, Hkv, D, 0, block_size, Lmax)
    _load().oracle_attend(ctypes.byref(dm), qp, kp_, vp, slp, ip, np_, int(kmax), float(sm_scale),
                          out.ctypes.data_as(ctypes.c_void_p), lse.ctypes.data_as(ctypes.c_void_p))
    return out, lse


def block_mass(q_bits, k_bits, seq_lens, block_size, sm_scale=0.0):
    """Block-level ground truth: each query head's dense softmax mass per KV block.

    q_bits uint16 [B, Hq, D]; k_bits uint16 [B, Hkv, Lmax, D]; seq_lens int32 [B].
    Returns (mass float64 [B, Hq, NBmax] (0 past NB_b), lse float64 [B, Hq]).
    """
    q_bits, qp = _c(q_bits, np.uint16)
    k_bits, kp_ = _c(k_bits, np.uint16)
    B, Hq, D = q_bits.shape
    _, Hkv, Lmax, _ = k_bits.shape
    sl, slp = _c(seq_lens, np.int32)
    nbmax = (Lmax + block_size - 1) // block_size
    mass = np.empty((B, Hq, nbmax), np.float64)
    lse = np.empty((B, Hq), np.float64)
    dm = _dims(B, Hq, Hkv, D, 0, block_size, Lmax)
    _load().oracle_block_mass(ctypes.byref(dm), qp, kp_, slp, float(sm_scale), mass.ctypes.data_as(ctypes.c_void_p),
                              lse.ctypes.data_as(ctypes.c_void_p))
    return mass, lse


def merge(o_parts, lse_parts):
    """Merge softmax partials over disjoint token sets: o_parts [n, D], lse_parts [n]."""
    o_parts, op = _c(o_parts, np.float64)
    lse_parts, lp = _c(lse_parts, np.float64)
    n, D = o_parts.shape
    out = np.empty(D, np.float64)
    lse = np.empty(1, np.float64)
    _load().oracle_merge(int(n), int(D), op, lp, out.ctypes.data_as(ctypes.c_void_p),
                         lse.ctypes.data_as(ctypes.c_void_p))
    return out, float(lse[0])


def step(q_bits, k_bits, v_bits, w_q, w_k, seq_lens, block_size, budget_tokens, sm_scale=0.0):
    """The whole decode step: pool -> gate -> select -> attend.

    Returns a dict with kpool, scores, block_idx, num_selected, out, lse.
    """
    Lmax = k_bits.shape[2]
    kpool = pool_project(k_bits, w_k, seq_lens, block_size)
    scores = gate_scores(q_bits, w_q, kpool, seq_lens, block_size, Lmax)
    idx, nsel = select_blocks(scores, seq_lens, block_size, Lmax, budget_tokens)
    out, lse = attend(q_bits, k_bits, v_bits, seq_lens, idx, nsel, block_size, sm_scale)
    return dict(kpool=kpool, scores=scores, block_idx=idx, num_selected=nsel, out=out, lse=lse)


def near_tie_rows(scores, block_idx, num_selected, seq_lens, block_size, threshold=1e-6):
    """Rows whose selection is decided by a gap below ``threshold``.

    For each (b, kvh) row with k_b - 1 >= 1 kept non-last blocks and at least
    one dropped block: gap = min kept non-last score - max dropped score. A
    row is a near tie when gap < threshold (absolute, on the oracle's score).
    Returns a bool array [B, Hkv].
    """
    B, Hkv, _ = scores.shape
    ties = np.zeros((B, Hkv), bool)
    for b in range(B):
        NB = num_blocks(int(seq_lens[b]), block_size)
        for h in range(Hkv):
            n = int(num_selected[b, h])
            kept = set(int(j) for j in block_idx[b, h, :n]) - {NB - 1}
            dropped = [j for j in range(NB - 1) if j not in kept]
            if not kept or not dropped:
                continue
            s = scores[b, h]
            gap = min(s[j] for j in kept) - max(s[j] for j in dropped)
            ties[b, h] = gap < threshold
    return ties
