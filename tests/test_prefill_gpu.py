"""Block-sparse prefill on the GPU against the oracle (attention on the tcgen05
tensor cores: two M = 128 query tiles per CTA, 64-token key sub-tiles).

* gate scores (query block i, key block j <= i < NB_b): |err| <= 2e-6 (an
  fp32 mean over the group's and the block's queries, one projection, a dot
  with the fp32 pooled keys);
* per-query-block lists: bit-exact with the oracle's selection run on the
  same fp32 scores (widened exactly);
* attention, given those lists: max |err| <= 1e-2, mean |err| <= 1e-3 (P is
  rounded to bf16 for the tensor-core P V, as in the decode), lse |err| <=
  1e-3; rows past the length 0 / -inf.
Cache and query padding past the length is NaN: it must never reach a result.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_seer_b200 import api
from oracle import oracle as O

pytestmark = pytest.mark.gpu


def make(B, Hq, Hkv, D, dg, blk, Lmax, lens, seed, pad=True):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, Lmax, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    if pad:
        for b, L in enumerate(lens):
            q[b, :, L:] = float("nan")
            k[b, :, L:] = float("nan")
            v[b, :, L:] = float("nan")
    wq = torch.randn(Hkv, dg, D, generator=g) / math.sqrt(D)
    wk = torch.randn(Hkv, dg, D, generator=g) / math.sqrt(D)
    return dict(q=q, k=k, v=v, w_q=wq, w_k=wk, lens=np.array(lens, np.int32), blk=blk)


def u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def run(c, budget, dense=False):
    B, Hq, Lmax, D = c["q"].shape
    Hkv, dg = c["w_q"].shape[0], c["w_q"].shape[1]
    blk = c["blk"]
    nbm = -(-Lmax // blk)
    dims = api.make_dims(B, Hq, Hkv, D, dg, blk, Lmax)
    dev = {n: c[n].cuda() for n in ("q", "k", "v", "w_q", "w_k")}
    lens = torch.from_numpy(c["lens"]).cuda()
    st = api.DecodeStep(B, Hq, Hkv, D, dg, blk, Lmax, budget_tokens=budget)
    st.build_pool(dev["k"], dev["w_k"], lens)
    scores = torch.full((B, Hkv, nbm, nbm), float("nan"), device="cuda")
    api.seer_prefill_gate_scores(dims, dev["q"], dev["w_q"], st.kpool, lens, scores)
    kmax = nbm if dense else budget // blk
    idx = torch.full((B, Hkv, nbm, kmax), -7, dtype=torch.int32, device="cuda")
    ns = torch.full((B, Hkv, nbm), -7, dtype=torch.int32, device="cuda")
    if dense:
        for i in range(nbm):
            idx[:, :, i, :i + 1] = torch.arange(i + 1, dtype=torch.int32, device="cuda")
            idx[:, :, i, i + 1:] = -1
        nb_b = torch.from_numpy(-(-c["lens"] // blk)).cuda()
        ns[:] = torch.where(torch.arange(nbm, device="cuda")[None, :] < nb_b[:, None],
                            torch.arange(1, nbm + 1, device="cuda")[None, :], 0).int()[:, None, :]
    else:
        api.seer_prefill_select_blocks(dims, scores, lens, budget, idx, ns)
    out = torch.empty(B, Hq, Lmax, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Hq, Lmax, device="cuda")
    api.seer_prefill_attention(dims, dev["q"], dev["k"], dev["v"], lens, idx, ns, kmax, out, lse)
    torch.cuda.synchronize()
    return scores.cpu().double().numpy(), idx.cpu().numpy(), ns.cpu().numpy(), out.cpu().double().numpy(), \
        lse.cpu().double().numpy()


def check(c, budget, dense=False):
    blk = c["blk"]
    g_s, g_idx, g_ns, g_out, g_lse = run(c, budget, dense)
    q, k, v = u16(c["q"]), u16(c["k"]), u16(c["v"])
    kp = O.pool_project(k, c["w_k"].numpy(), c["lens"], blk)
    o_s = O.prefill_gate(q, c["w_q"].numpy(), kp, c["lens"], blk)
    for b, L in enumerate(int(x) for x in c["lens"]):
        NB = -(-L // blk)
        for i in range(NB):
            err = np.abs(g_s[b, :, i, :i + 1] - o_s[b, :, i, :i + 1]).max()
            assert err <= 2e-6, (b, i, err)
    if not dense:
        Lmax = c["q"].shape[2]
        r_idx, r_ns = O.prefill_select(g_s, c["lens"], blk, Lmax, budget)
        np.testing.assert_array_equal(g_ns, r_ns)
        np.testing.assert_array_equal(g_idx, r_idx)
    o_out, o_lse = O.prefill_attend(q, k, v, c["lens"], g_idx, g_ns, blk)
    for b, L in enumerate(int(x) for x in c["lens"]):
        d = np.abs(g_out[b, :, :L] - o_out[b, :, :L])
        if L:
            assert d.max() <= 1e-2 and d.mean() <= 1e-3, (d.max(), d.mean())
            assert np.abs(g_lse[b, :, :L] - o_lse[b, :, :L]).max() <= 1e-3
        assert np.all(g_out[b, :, L:] == 0.0) and np.all(g_lse[b, :, L:] == -np.inf)


@pytest.mark.parametrize("shape", [
    (2, 8, 2, 128, 128, 64, 512, [512, 301], 128),
    (2, 8, 2, 128, 64, 128, 768, [768, 130], 256),
    (1, 4, 1, 64, 64, 64, 448, [448], 64),
    (3, 4, 2, 64, 128, 128, 512, [512, 0, 129], 128),
    (1, 10, 2, 128, 128, 64, 1024, [1000], 256),
    (2, 2, 2, 128, 128, 64, 512, [400, 512], 128),      # one head per group: half an M tile
    (1, 8, 1, 128, 64, 64, 640, [640], 192),            # eight heads: two CTAs per query block
    (2, 4, 2, 128, 128, 64, 500, [500, 77], 128),       # Lmax not a multiple of the block
    (1, 4, 1, 64, 64, 128, 640, [577], 256),            # D 64, blk 128, a ragged last block
])
def test_prefill_matches_oracle(shape):
    B, Hq, Hkv, D, dg, blk, Lmax, lens, budget = shape
    check(make(B, Hq, Hkv, D, dg, blk, Lmax, lens, seed=len(lens) + Lmax), budget)


@pytest.mark.parametrize("blk", [64, 128])
def test_prefill_dense_lists(blk):
    check(make(2, 4, 2, 128, 128, blk, 512, [512, 333], seed=blk), budget=blk, dense=True)


def attend_lists(c, lists, kmax):
    """The prefill attention on given per-query-block lists, against the oracle on the same lists."""
    B, Hq, Lmax, D = c["q"].shape
    Hkv = c["k"].shape[1]
    blk = c["blk"]
    nbm = -(-Lmax // blk)
    idx = np.full((B, Hkv, nbm, kmax), -1, np.int32)
    ns = np.zeros((B, Hkv, nbm), np.int32)
    for i, lst in enumerate(lists):
        idx[:, :, i, :len(lst)] = lst
        ns[:, :, i] = len(lst)
    dims = api.make_dims(B, Hq, Hkv, D, 128, blk, Lmax)
    out = torch.empty(B, Hq, Lmax, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Hq, Lmax, device="cuda")
    lens = torch.from_numpy(c["lens"]).cuda()
    api.seer_prefill_attention(dims, c["q"].cuda(), c["k"].cuda(), c["v"].cuda(), lens, torch.from_numpy(idx).cuda(),
                               torch.from_numpy(ns).cuda(), kmax, out, lse)
    torch.cuda.synchronize()
    o_out, o_lse = O.prefill_attend(u16(c["q"]), u16(c["k"]), u16(c["v"]), c["lens"], idx, ns, blk)
    g_out, g_lse = out.cpu().double().numpy(), lse.cpu().double().numpy()
    L = int(c["lens"][0])
    d = np.abs(g_out[0, :, :L] - o_out[0, :, :L])
    # the output is bf16: a token that sees one or two keys returns a V row of magnitude up to
    # ~5, where half a bf16 unit in the last place is 2^-6; the bound adds that rounding
    bound = 1e-2 + 2.0 ** -7 * np.abs(o_out[0, :, :L])
    assert np.all(d <= bound), (d.max(), (d - bound).max())
    assert d.mean() <= 1e-3, d.mean()
    assert np.abs(g_lse[0, :, :L] - o_lse[0, :, :L]).max() <= 1e-3
    return g_out, o_out


def late_lists(nb, late, keep, rng):
    """Each query block keeps only itself, except the last `late`, which keep `keep` blocks:
    themselves and keep - 1 earlier ones drawn at random (ascending lists)."""
    lists = []
    for i in range(nb):
        if i < nb - late:
            lists.append([i])
        else:
            lists.append(sorted(rng.choice(i, size=keep - 1, replace=False).tolist()) + [i])
    return lists


def test_prefill_deep_lists_wrap_the_rings():
    # an 8K-token prompt; the last three query blocks keep 64 blocks (a 4K-token budget):
    # 32 key sub-tiles per query tile, so the 2-slot K ring and the 3-slot V ring wrap
    # 16 and 10 times
    c = make(1, 4, 1, 128, 128, 64, 8192, [8192], seed=81)
    rng = np.random.default_rng(81)
    attend_lists(c, late_lists(128, 3, 64, rng), 64)


def test_prefill_late_salient_block_rescales():
    # the last three query blocks keep 64 blocks; in each list, the last earlier block
    # has its keys scaled x8 (exact in bf16), so a row's maximum grows by far more than
    # 2^8 after the first sub-tiles and the running output and sum are rescaled
    c = make(1, 4, 1, 128, 128, 64, 8192, [8192], seed=82)
    rng = np.random.default_rng(82)
    lists = late_lists(128, 3, 64, rng)
    for lst in lists[-3:]:
        j = lst[-2]
        c["k"][:, :, j * 64:(j + 1) * 64] = (c["k"][:, :, j * 64:(j + 1) * 64].float() * 8).to(torch.bfloat16)
    g_out, _ = attend_lists(c, lists, 64)
    assert np.isfinite(g_out[0, :, -192:]).all()


def test_prefill_lists_longer_than_the_staged_limit():
    # 400 blocks of 64: the last two query blocks keep every block (399 and 400 entries, more
    # than the 384 list entries a CTA stages in shared memory), read from global memory
    c = make(1, 4, 1, 128, 128, 64, 64 * 400, [64 * 400], seed=83)
    lists = [[i] for i in range(398)] + [list(range(399)), list(range(400))]
    attend_lists(c, lists, 400)
