"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Small shapes are checked everywhere (they span several tiles, ragged tails,
every supported head_dim / block size / group size); the workload sizes the
benchmark times are checked on sampled batch entries the oracle computes one
by one, in the same launch configuration (DecodeStep, default split count).
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_seer_b200 import api
from block_sparse_attention_seer_b200 import workloads as W
from oracle import oracle as O

from gpu_helpers import (check_attention, check_indices, check_kpool, check_scores, gpu_attend, gpu_step,
                         oracle_bits, to_dev)

pytestmark = pytest.mark.gpu


def full_chain(wl, inp, batches=None, num_splits=None, expect_no_ties=False):
    """GPU step vs oracle step on `batches` (all when None). Returns (excluded rows, max err, mean err)."""
    st, g = gpu_step(inp, wl, num_splits)
    c = oracle_bits(inp, batches)
    ora = O.step(c["q"], c["k"], c["v"], c["w_q"], c["w_k"], c["lens"], wl.block_size, wl.budget_tokens)
    sel = slice(None) if batches is None else list(batches)
    check_kpool(g["kpool"][sel], ora["kpool"], c["lens"], wl.block_size)
    check_scores(g["scores"][sel], ora["scores"], c["lens"], wl.block_size)
    excluded = check_indices(g["block_idx"][sel], g["num_selected"][sel], ora["block_idx"], ora["num_selected"],
                             ora["scores"], c["lens"], wl.block_size)
    if expect_no_ties:
        assert excluded == 0
    # attention given the oracle's block lists
    idx = g["block_idx"].copy()
    ns = g["num_selected"].copy()
    idx[sel] = ora["block_idx"]
    ns[sel] = ora["num_selected"]
    out, lse = gpu_attend(st, inp, idx, ns, num_splits)
    mx, mean = check_attention(out[sel], lse[sel], ora["out"], ora["lse"])
    return excluded, mx, mean


# ---------------------------------------------------------------- small shapes, whole batch

@pytest.mark.parametrize("seed", range(10))
def test_tiny_workload(seed):
    wl = W.WORKLOADS["tiny"]
    inp = to_dev(W.make_inputs(wl, seed=seed))
    full_chain(wl, inp)


SHAPES = {
    # name: (B, Hq, Hkv, D, dg, blk, Lmax, lens, budget)
    "d128_b64_g4_ragged": (3, 32, 8, 128, 128, 64, 4096, [4096, 3001, 1], 1024),
    "d128_b128_g5": (2, 40, 8, 128, 128, 128, 8192, [8192, 5000], 1280),
    "d64_b128_g8_dg128": (2, 8, 1, 64, 128, 128, 2048, [2000, 129], 512),
    "d64_b64_g1": (4, 2, 2, 64, 64, 64, 1024, [64, 65, 127, 1000], 256),
    "d128_b64_g2_dg64": (2, 4, 2, 128, 64, 64, 3000, [2999, 1500], 640),
}


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_small_shapes_nan_padded(name):
    B, Hq, Hkv, D, dg, blk, Lmax, lens, budget = SHAPES[name]
    wl = W.Workload(name, B, Hq, Hkv, D, dg, blk, Lmax, budget)
    inp = to_dev(W.make_inputs(wl, seed=11, pad_value=float("nan"), seq_lens=np.array(lens, np.int32)))
    full_chain(wl, inp)


@pytest.mark.parametrize("num_splits", [1, 2, 7, None])
def test_split_count_does_not_change_result(num_splits):
    B, Hq, Hkv, D, dg, blk, Lmax, lens, budget = SHAPES["d128_b64_g4_ragged"]
    wl = W.Workload("splits", B, Hq, Hkv, D, dg, blk, Lmax, budget)
    inp = to_dev(W.make_inputs(wl, seed=3, seq_lens=np.array(lens, np.int32)))
    full_chain(wl, inp, num_splits=num_splits)


def test_dense_block_list_small():
    B, Hq, Hkv, D, dg, blk, Lmax, lens, budget = SHAPES["d128_b128_g5"]
    wl = W.Workload("dense", B, Hq, Hkv, D, dg, blk, Lmax, budget)
    inp = to_dev(W.make_inputs(wl, seed=4, pad_value=float("nan"), seq_lens=np.array(lens, np.int32)))
    st = api.DecodeStep(**wl.dims(), budget_tokens=budget)
    idx, ns = W.identity_block_list(inp["seq_lens_host"], Hkv, blk, wl.nb_max)
    out, lse = gpu_attend(st, inp, idx, ns)
    c = oracle_bits(inp)
    o, l = O.attend(c["q"], c["k"], c["v"], c["lens"], idx, ns, blk)
    check_attention(out, lse, o, l)


# ---------------------------------------------------------------- edge cases

def test_edge_lengths_budget_and_bad_indices():
    # empty row (L=0), one token, exactly one full block, budget >= L, kmax = 1
    wl = W.Workload("edge", 5, 8, 2, 128, 128, 64, 512, 64)
    lens = np.array([0, 1, 64, 512, 300], np.int32)
    inp = to_dev(W.make_inputs(wl, seed=5, pad_value=float("nan"), seq_lens=lens))
    full_chain(wl, inp)                       # kmax = 1: only the last block
    for budget in (512, 4096):                # every block kept
        full_chain(wl.with_(budget_tokens=budget), inp)
    st, g = gpu_step(inp, wl.with_(budget_tokens=256))
    assert (g["out"][0] == 0).all() and np.isneginf(g["lse"][0]).all()
    assert (g["num_selected"][0] == 0).all()
    # indices outside [0, NB_b) are skipped
    idx = np.array([[[0, -1, 9]] * 2, [[0, 5, -7]] * 2, [[0, 3, 1]] * 2, [[7, 2, 100]] * 2, [[4, 2, 0]] * 2],
                   np.int32)
    ns = np.full((5, 2), 3, np.int32)
    out, lse = gpu_attend(st, inp, idx, ns)
    clean = np.where((idx >= 0) & (idx < np.array([0, 1, 1, 8, 5])[:, None, None]), idx, -1)
    c = oracle_bits(inp)
    o, l = O.attend(c["q"], c["k"], c["v"], c["lens"], clean, ns, 64)
    check_attention(out, lse, o, l)


def test_decode_refresh_matches_bulk_pool():
    wl = W.Workload("refresh", 2, 8, 2, 128, 128, 64, 1024, 256)
    lens = np.array([1000, 700], np.int32)
    inp = to_dev(W.make_inputs(wl, seed=6, seq_lens=lens))
    st = api.DecodeStep(**wl.dims(), budget_tokens=256)
    st.build_pool(inp["k_cache"], inp["w_k"], inp["seq_lens"])
    # append one token per sequence, then refresh only the open block
    new_lens = inp["seq_lens"] + 1
    inp["k_cache"][0, :, 1000] = torch.randn(2, 128, device="cuda").bfloat16()
    inp["k_cache"][1, :, 700] = torch.randn(2, 128, device="cuda").bfloat16()
    st.set_update_start(new_lens)
    api.seer_kpool_update(st.dims, inp["k_cache"], inp["w_k"], new_lens, st.upd_start, st.kpool)
    ref = api.DecodeStep(**wl.dims(), budget_tokens=256)
    ref.build_pool(inp["k_cache"], inp["w_k"], new_lens)
    torch.cuda.synchronize()
    for b, L in enumerate((1001, 701)):
        nb = -(-L // 64)
        assert torch.equal(st.kpool[b, :, :nb], ref.kpool[b, :, :nb])


# ---------------------------------------------------------------- full workload sizes, sampled

@pytest.mark.parametrize("name,batches", [
    ("decode_b16", [0, 15]),
    ("large_block", [0, 7]),
    ("ragged", [0, 63]),
    ("sweep_b4_keep05", [3]),
])
def test_full_size_sampled(name, batches):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, seed=0, device="cuda", pad_value=float("nan") if wl.ragged else None)
    excluded, mx, mean = full_chain(wl, inp, batches=batches)
    print(f"{name}: near-tie rows excluded {excluded}, out max {mx:.2e} mean {mean:.2e}")


def test_full_size_sweep_b1_whole_batch():
    wl = W.WORKLOADS["sweep_b1_keep10"]
    inp = W.make_inputs(wl, seed=0, device="cuda")
    full_chain(wl, inp)


@pytest.mark.parametrize("name,batches", [("decode_b16", [9]), ("sweep_b1_dense", None)])
def test_full_size_dense_block_list(name, batches):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, seed=1, device="cuda")
    st = api.DecodeStep(**wl.dims(), budget_tokens=wl.budget_tokens)
    idx, ns = W.identity_block_list(inp["seq_lens_host"], wl.num_kv_heads, wl.block_size, wl.nb_max)
    out, lse = gpu_attend(st, inp, idx, ns)
    sel = slice(None) if batches is None else batches
    c = oracle_bits(inp, batches)
    o, l = O.attend(c["q"], c["k"], c["v"], c["lens"], idx[sel], ns[sel], wl.block_size)
    check_attention(out[sel], lse[sel], o, l)
