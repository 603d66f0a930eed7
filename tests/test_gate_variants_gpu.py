"""Gate variants against the oracle: per-head scores aggregated by mean, max or
softmax mean (seer_gate_scores_agg), and threshold selection
(seer_select_blocks_threshold).

Tolerances: mean and max scores |err| <= 2e-6 (each head's fp32 score of
fp32 pooled keys, as the mean gate's 1e-6 with the per-head rounding on top);
softmax mean |err| <= 1e-8 + 1e-5 * value (a score error of ~1e-6 moves
exp(s - lse) by a relative ~2e-6). The threshold selection runs on the same
fp32 scores on both sides (widened exactly for the oracle), so its lists are
compared bit for bit, ties and scores equal to the threshold included.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_seer_b200 import api
from block_sparse_attention_seer_b200 import workloads as W
from oracle import oracle as O

from gpu_helpers import oracle_bits

pytestmark = pytest.mark.gpu


def gpu_scores(wl, inp, agg):
    dims = api.make_dims(**wl.dims())
    st = api.DecodeStep(**wl.dims(), budget_tokens=wl.budget_tokens)
    st.build_pool(inp["k_cache"], inp["w_k"], inp["seq_lens"])
    s = torch.full((wl.batch, wl.num_kv_heads, wl.nb_max), float("nan"), dtype=torch.float32, device="cuda")
    api.seer_gate_scores_agg(dims, inp["q"], inp["w_q"], st.kpool, inp["seq_lens"], agg, s)
    torch.cuda.synchronize()
    return s.cpu().double().numpy()


def check_agg(wl, inp, agg, batches=None):
    got = gpu_scores(wl, inp, agg)
    sel = list(range(wl.batch)) if batches is None else list(batches)
    c = oracle_bits(inp, sel if batches is not None else None)
    kp = O.pool_project(c["k"], c["w_k"], c["lens"], wl.block_size)
    ref = O.gate_scores_agg(c["q"], c["w_q"], kp, c["lens"], wl.block_size, wl.max_seq_len, agg)
    worst = 0.0
    for i, b in enumerate(sel):
        nb = -(-int(c["lens"][i]) // wl.block_size)
        g, r = got[b, :, :nb], ref[i, :, :nb]
        tol = 2e-6 if agg != O.AGG_SOFTMAX_MEAN else 1e-8 + 1e-5 * np.abs(r)
        assert np.all(np.abs(g - r) <= tol), np.abs(g - r).max()
        worst = max(worst, float(np.abs(g - r).max()) if nb else 0.0)
        if agg == O.AGG_SOFTMAX_MEAN and nb:
            assert np.all(np.abs(g.sum(-1) - 1.0) <= 1e-5)
    return worst


@pytest.mark.parametrize("agg", [0, 1, 2])
@pytest.mark.parametrize("seed", range(2))
def test_aggregations_tiny(agg, seed):
    wl = W.WORKLOADS["tiny"]
    check_agg(wl, W.make_inputs(wl, seed=seed, device="cuda"), agg)


@pytest.mark.parametrize("agg", [0, 1, 2])
@pytest.mark.parametrize("shape", [
    (3, 32, 8, 128, 128, 64, 4096, [4096, 3001, 1]),
    (2, 40, 8, 128, 64, 128, 8192, [8192, 5000]),
    (2, 8, 1, 64, 128, 128, 2048, [2000, 129]),
    (5, 8, 2, 64, 64, 64, 512, [0, 1, 64, 512, 300]),
])
def test_aggregations_small_shapes(agg, shape):
    B, Hq, Hkv, D, dg, blk, Lmax, lens = shape
    wl = W.Workload("agg", B, Hq, Hkv, D, dg, blk, Lmax, blk)
    check_agg(wl, W.make_inputs(wl, seed=6, device="cuda", seq_lens=np.array(lens, np.int32)), agg)


@pytest.mark.parametrize("agg", [1, 2])
def test_aggregations_full_size_sampled(agg):
    wl = W.WORKLOADS["decode_b16"]
    err = check_agg(wl, W.make_inputs(wl, seed=0, device="cuda"), agg, batches=[0, 15])
    print(f"aggregation {agg} at decode_b16: max abs error {err:.2e}")


def run_threshold(scores_f32, lens, blk, Lmax, budget, tau):
    B, Hkv, _ = scores_f32.shape
    dims = api.make_dims(B, Hkv, Hkv, 128, 128, blk, Lmax)
    kmax = budget // blk
    s = torch.from_numpy(scores_f32).cuda()
    sl = torch.from_numpy(np.asarray(lens, np.int32)).cuda()
    idx = torch.full((B, Hkv, kmax), -7, dtype=torch.int32, device="cuda")
    ns = torch.full((B, Hkv), -7, dtype=torch.int32, device="cuda")
    api.seer_select_blocks_threshold(dims, s, sl, budget, tau, idx, ns)
    torch.cuda.synchronize()
    ref_idx, ref_ns = O.select_threshold(scores_f32.astype(np.float64), np.asarray(lens, np.int32), blk, Lmax, budget,
                                         float(np.float32(tau)))
    np.testing.assert_array_equal(ns.cpu().numpy(), ref_ns)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)


@pytest.mark.parametrize("nb,blk,budget_blocks", [(2, 64, 1), (33, 64, 8), (512, 64, 64), (1024, 128, 103),
                                                  (4097, 64, 512)])
def test_threshold_selection_matches_oracle(nb, blk, budget_blocks):
    rng = np.random.default_rng(nb)
    B, Hkv, Lmax = 2, 3, nb * blk
    scores = np.round(rng.standard_normal((B, Hkv, nb)), 2).astype(np.float32)  # ties, some equal to tau
    lens = [Lmax, max(1, Lmax - blk // 2 - blk * (nb // 3))]
    for tau in (-np.inf, np.inf, 0.0, 1.0, float(scores[0, 0, 0]), -0.5):
        run_threshold(scores, lens, blk, Lmax, budget_blocks * blk, tau)
