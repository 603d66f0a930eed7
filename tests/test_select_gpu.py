"""seer_select_blocks on adversarial scores: the kept lists must equal the
oracle's selection on the same fp32 scores (widened exactly to fp64) bit for
bit -- including all-equal scores (lowest indices win), clusters within a few
ulps (the value histogram narrows its key range over several steps), few
distinct values, duplicated values at the boundary and signed zeros. The
select (select_row) builds a histogram of the candidates' order keys over
their value range, scans it from the top to the bin that holds the last
kept key, ranks that bin exactly when it is small and narrows the range to
it otherwise; the sizes run from 1 to 4096 candidates.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_seer_b200 import api
from oracle import oracle as O

pytestmark = pytest.mark.gpu


def run(scores_f32, lens, blk, Lmax, budget):
    B, Hkv, NBmax = scores_f32.shape
    dims = api.make_dims(B, Hkv, Hkv, 128, 128, blk, Lmax)
    kmax = budget // blk
    s = torch.from_numpy(scores_f32).cuda()
    sl = torch.from_numpy(np.asarray(lens, np.int32)).cuda()
    idx = torch.full((B, Hkv, kmax), -7, dtype=torch.int32, device="cuda")
    ns = torch.zeros(B, Hkv, dtype=torch.int32, device="cuda")
    api.seer_select_blocks(dims, s, sl, budget, idx, ns)
    torch.cuda.synchronize()
    ref_idx, ref_ns = O.select_blocks(scores_f32.astype(np.float64), np.asarray(lens, np.int32), blk, Lmax, budget)
    np.testing.assert_array_equal(ns.cpu().numpy(), ref_ns)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)


CASES = {
    "normal": lambda rng, n: rng.standard_normal(n).astype(np.float32) * 0.06,
    "all_equal": lambda rng, n: np.full(n, 0.25, np.float32),
    "clustered": lambda rng, n: (0.5 + rng.integers(0, 40, n) * 1e-7).astype(np.float32),
    "few_values": lambda rng, n: rng.choice(np.array([0.1, 0.2, 0.3, -0.2], np.float32), n),
    "signed_zeros": lambda rng, n: rng.choice(np.array([0.0, -0.0, 1e-30, -1e-30], np.float32), n),
    "wide": lambda rng, n: (rng.standard_normal(n) * 10.0 ** rng.integers(-20, 20, n)).astype(np.float32),
    # powers of two over many octaves: the key range narrows over several histogram steps
    "geometric": lambda rng, n: (rng.choice([-1.0, 1.0], n) * 2.0 ** -rng.integers(0, 120, n)).astype(np.float32),
    # a dense run of adjacent floats next to a few far outliers
    "adjacent_ulps": lambda rng, n: np.where(rng.random(n) < 0.02, 1e30,
                                             1.0 + rng.integers(0, 3 * n, n) * 2.0 ** -23).astype(np.float32),
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("nb,blk,budget_blocks", [(2, 64, 1), (33, 64, 8), (512, 64, 64), (513, 64, 100),
                                                  (514, 64, 100), (1024, 128, 103), (1025, 64, 300),
                                                  (1026, 64, 700), (2049, 64, 300), (2050, 64, 1000),
                                                  (4097, 64, 512)])
def test_select_matches_oracle(case, nb, blk, budget_blocks):
    rng = np.random.default_rng(nb * 7 + len(case))
    B, Hkv = 2, 3
    Lmax = nb * blk
    scores = np.stack([np.stack([CASES[case](rng, nb) for _ in range(Hkv)]) for _ in range(B)])
    lens = [Lmax, max(1, Lmax - blk // 2 - blk * (nb // 3))]
    run(scores, lens, blk, Lmax, budget_blocks * blk)
