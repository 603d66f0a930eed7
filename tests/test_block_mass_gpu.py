"""seer_block_mass (the gate's block-level ground truth) against the oracle.

Tolerance, from the arithmetic: a logit is an fp32 sum of D exact bf16
products (tensor-core accumulate), so its error stays within a few 1e-5 after
the 1/sqrt(D) scale; mass_j = exp(blse_j - lse) then carries a relative error
of about 1e-4. Checked: |mass - oracle| <= 5e-5 + 1e-4 * oracle, |lse -
oracle| <= 1e-4, blocks past the length exactly 0, every row summing to 1.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_seer_b200 import api
from block_sparse_attention_seer_b200 import workloads as W
from oracle import oracle as O

pytestmark = pytest.mark.gpu


def run_mass(wl, inp):
    dims = api.make_dims(**wl.dims())
    mass = torch.full((wl.batch, wl.num_q_heads, wl.nb_max), -7.0, dtype=torch.float32, device="cuda")
    lse = torch.empty(wl.batch, wl.num_q_heads, dtype=torch.float32, device="cuda")
    api.seer_block_mass(dims, inp["q"], inp["k_cache"], inp["seq_lens"], mass, lse)
    torch.cuda.synchronize()
    return mass.cpu().double().numpy(), lse.cpu().double().numpy()


def check(wl, inp, batches=None):
    mass, lse = run_mass(wl, inp)
    sel = list(range(wl.batch)) if batches is None else list(batches)
    q = W.bf16_bits(inp["q"].cpu())[sel]
    k = W.bf16_bits(inp["k_cache"].cpu())[sel]
    lens = inp["seq_lens_host"][sel]
    ref_m, ref_l = O.block_mass(q, k, lens, wl.block_size)
    got_m, got_l = mass[sel], lse[sel]
    assert np.all(np.abs(got_m - ref_m) <= 5e-5 + 1e-4 * ref_m), np.abs(got_m - ref_m).max()
    live = np.isfinite(ref_l)
    assert np.all(np.abs(got_l[live] - ref_l[live]) <= 1e-4)
    assert np.all(got_l[~live] == -np.inf)
    for i, L in enumerate(lens):
        nb = -(-int(L) // wl.block_size)
        assert np.all(got_m[i, :, nb:] == 0.0)
        if L > 0:
            assert np.all(np.abs(got_m[i].sum(-1) - 1.0) <= 1e-4)
    return np.abs(got_m - ref_m).max()


@pytest.mark.parametrize("seed", range(3))
def test_block_mass_tiny(seed):
    wl = W.WORKLOADS["tiny"]
    inp = W.make_inputs(wl, seed=seed, device="cuda")
    check(wl, inp)


@pytest.mark.parametrize("shape", [
    (3, 32, 8, 128, 128, 64, 4096, [4096, 3001, 1]),
    (2, 40, 8, 128, 128, 128, 8192, [8192, 5000]),
    (2, 8, 1, 64, 128, 128, 2048, [2000, 129]),
    (4, 2, 2, 64, 64, 64, 1024, [64, 65, 127, 1000]),
    (5, 8, 2, 128, 128, 64, 512, [0, 1, 64, 512, 300]),
])
def test_block_mass_small_shapes(shape):
    B, Hq, Hkv, D, dg, blk, Lmax, lens = shape
    wl = W.Workload("mass", B, Hq, Hkv, D, dg, blk, Lmax, blk)
    inp = W.make_inputs(wl, seed=4, device="cuda", pad_value=float("nan"), seq_lens=np.array(lens, np.int32))
    check(wl, inp)


@pytest.mark.parametrize("name,batches", [("decode_b16", [0, 15]), ("ragged", [0, 63]), ("large_block", [5])])
def test_block_mass_full_size_sampled(name, batches):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, seed=0, device="cuda", pad_value=float("nan") if wl.ragged else None)
    err = check(wl, inp, batches)
    print(f"block mass {name}: max abs error {err:.2e}")
