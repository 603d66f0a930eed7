"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test fixes one part of the method against a closed form, a hand-derived
example, a library routine the oracle does not call, an invariant, or brute
force, so that a dropped term, a wrong sign or index, or a transposed operand
anywhere in the oracle fails at least one of them.

Method sources: "SeerAttention-R: Sparse Attention Adaptation for Long
Reasoning" (abstract) and "SeerAttention: Learning Intrinsic Sparse Attention
in Your LLMs" (abstract).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from block_sparse_attention_seer_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits(a) -> np.ndarray:
    """bf16 bit patterns of exactly representable values (checked)."""
    t = torch.as_tensor(np.asarray(a, np.float32))
    b = t.to(torch.bfloat16)
    assert torch.equal(b.float(), t), "value not exact in bf16"
    return b.view(torch.int16).numpy().view(np.uint16)


def widen(u16: np.ndarray) -> np.ndarray:
    return torch.from_numpy(u16.view(np.int16)).view(torch.bfloat16).double().numpy()


def small_case(seed, B=2, Hq=4, Hkv=2, D=64, dg=64, blk=64, Lmax=320, lens=(320, 257), budget=128):
    wl = W.Workload("pin", B, Hq, Hkv, D, dg, blk, Lmax, budget)
    inp = W.make_inputs(wl, seed=seed, seq_lens=np.array(lens, np.int32))
    return wl, dict(q=W.bf16_bits(inp["q"]), k=W.bf16_bits(inp["k_cache"]),
                    v=W.bf16_bits(inp["v_cache"]), w_q=inp["w_q"].numpy(), w_k=inp["w_k"].numpy(),
                    lens=inp["seq_lens_host"])


# ---------------------------------------------------------------- gate: pool, project, score

def test_toy_gate_matches_hand_derivation(oracle):
    g = json.load(open(os.path.join(GOLDEN, "toy_gate.json")))
    dm = g["dims"]
    K = bits(np.array(g["K"], np.float32))[None, None]            # [1,1,6,4]
    q = bits(np.array(g["q"], np.float32))[None]                  # [1,2,4]
    wk = np.array(g["W_k"], np.float32)[None]
    wq = np.array(g["W_q"], np.float32)[None]
    lens = np.array([g["seq_len"]], np.int32)
    kp = oracle.pool_project(K, wk, lens, dm["block_size"])
    np.testing.assert_array_equal(kp[0, 0], np.array(g["kpool"], np.float64))
    s = oracle.gate_scores(q, wq, kp, lens, dm["block_size"], dm["max_seq_len"])
    np.testing.assert_allclose(s[0, 0], g["scores"], rtol=0, atol=1e-13)
    for budget, expect in g["selection"].items():
        idx, nsel = oracle.select_blocks(s, lens, dm["block_size"], dm["max_seq_len"], int(budget))
        assert list(idx[0, 0, :nsel[0, 0]]) == expect


def test_pool_closed_form_partial_block(oracle):
    # K[t, d] = (t mod 7) for even d, -(t mod 5) for odd d: exact in bf16; the
    # pooled mean of a block is the mean of those integers over its valid
    # tokens only (the partial last block divides by its own count).
    blk, D, dg, Lmax = 8, 16, 16, 40
    L = 29                                                       # NB = 4, last block has 5 tokens
    t = np.arange(Lmax)
    Kf = np.empty((Lmax, D), np.float32)
    Kf[:, 0::2] = (t % 7)[:, None]
    Kf[:, 1::2] = -(t % 5)[:, None]
    K = bits(Kf)[None, None]
    # W_k = cyclic shift by 3: kpool[e] = pooled[(e + 3) % D]
    wk = np.zeros((1, dg, D), np.float32)
    for e in range(dg):
        wk[0, e, (e + 3) % D] = 1.0
    kp = oracle.pool_project(K, wk, np.array([L], np.int32), blk)
    for j in range(4):
        toks = range(j * blk, min((j + 1) * blk, L))
        n = len(toks)
        even = sum(tt % 7 for tt in toks) / n
        odd = -sum(tt % 5 for tt in toks) / n
        pooled = np.array([even if d % 2 == 0 else odd for d in range(D)])
        np.testing.assert_allclose(kp[0, 0, j], [pooled[(e + 3) % D] for e in range(dg)], rtol=0, atol=1e-15)
    assert np.isnan(kp[0, 0, 4]).all()                            # block past NB is undefined


def test_score_identity_weights_closed_form(oracle):
    # W_q = W_k = I and dg = D: s_j = mean_h(q_h) . mean(K_block j) / sqrt(D)
    wl, c = small_case(1)
    D = wl.head_dim
    eye = np.broadcast_to(np.eye(D, dtype=np.float32), (wl.num_kv_heads, D, D)).copy()
    kp = oracle.pool_project(c["k"], eye, c["lens"], wl.block_size)
    s = oracle.gate_scores(c["q"], eye, kp, c["lens"], wl.block_size, wl.max_seq_len)
    q = widen(c["q"])
    K = widen(c["k"])
    G = wl.group
    for b in range(wl.batch):
        L = int(c["lens"][b])
        for h in range(wl.num_kv_heads):
            qbar = q[b, h * G:(h + 1) * G].mean(0)
            for j in range(-(-L // wl.block_size)):
                kbar = K[b, h, j * wl.block_size:min((j + 1) * wl.block_size, L)].mean(0)
                assert abs(s[b, h, j] - qbar @ kbar / math.sqrt(D)) < 1e-12


def test_gqa_mean_is_linear(oracle):
    # The mean over heads of per-head scores equals the score of the mean
    # projected query (linearity), checked with torch's float64 matmul.
    wl, c = small_case(2)
    kp = oracle.pool_project(c["k"], c["w_k"], c["lens"], wl.block_size)
    s = oracle.gate_scores(c["q"], c["w_q"], kp, c["lens"], wl.block_size, wl.max_seq_len)
    q = torch.from_numpy(widen(c["q"]))
    wq = torch.from_numpy(c["w_q"].astype(np.float64))
    G = wl.group
    for b in range(wl.batch):
        nb = -(-int(c["lens"][b]) // wl.block_size)
        for h in range(wl.num_kv_heads):
            qg_mean = (wq[h] @ q[b, h * G:(h + 1) * G].T).mean(1)
            ref = torch.from_numpy(kp[b, h, :nb]) @ qg_mean / math.sqrt(wl.gate_dim)
            np.testing.assert_allclose(s[b, h, :nb], ref.numpy(), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- selection

def test_topk_brute_force_tiny(oracle):
    # Tiny workload: NB=32, k=8. The 7 kept non-last blocks must maximise the
    # summed score over all C(31,7) = 2,629,575 subsets of blocks 0..30.
    wl = W.WORKLOADS["tiny"]
    combos = np.fromiter(itertools.chain.from_iterable(itertools.combinations(range(31), 7)),
                         dtype=np.int8, count=2629575 * 7).reshape(-1, 7)
    for seed in range(2):
        inp = W.make_inputs(wl, seed=seed)
        st = oracle.step(W.bf16_bits(inp["q"]), W.bf16_bits(inp["k_cache"]), W.bf16_bits(inp["v_cache"]),
                         inp["w_q"].numpy(), inp["w_k"].numpy(), inp["seq_lens_host"], wl.block_size,
                         wl.budget_tokens)
        s = st["scores"][0, 0]
        sums = s[combos].sum(1)
        best = combos[np.argmax(sums)]
        kept = st["block_idx"][0, 0, :st["num_selected"][0, 0]]
        assert st["num_selected"][0, 0] == 8
        assert kept[-1] == 31
        assert sorted(best.tolist()) == kept[:-1].tolist()
        # and against numpy's lexsort (score descending, then index ascending)
        order = np.lexsort((np.arange(31), -s[:31]))
        assert sorted(order[:7].tolist()) == kept[:-1].tolist()


def test_last_block_always_kept_and_sizes(oracle):
    rng = np.random.default_rng(5)
    for trial in range(20):
        blk = [64, 128][trial % 2]
        lens = rng.integers(1, 3000, size=3).astype(np.int32)
        Lmax = int(lens.max()) + int(rng.integers(0, 200))
        nbm = -(-Lmax // blk)
        scores = rng.standard_normal((3, 2, nbm))
        budget = blk * int(rng.integers(1, 12))
        idx, nsel = oracle.select_blocks(scores, lens, blk, Lmax, budget)
        for b in range(3):
            nb = -(-int(lens[b]) // blk)
            kb = min(budget // blk, nb)
            for h in range(2):
                row = idx[b, h]
                assert nsel[b, h] == kb
                kept = row[:kb]
                assert kept[-1] == nb - 1                         # last block, and ascending order
                assert (np.diff(kept) > 0).all()
                assert (row[kb:] == -1).all()
                others = np.setdiff1d(np.arange(nb - 1), kept)
                if kb > 1 and len(others):
                    assert scores[b, h, kept[:-1]].min() >= scores[b, h, others].max()


def test_ties_go_to_lower_index(oracle):
    lens = np.array([1000], np.int32)
    scores = np.zeros((1, 1, 16))
    scores[0, 0, 9] = 1.0                                          # one clear winner, rest tied
    idx, nsel = oracle.select_blocks(scores, lens, 64, 1000, 64 * 5)
    assert idx[0, 0, :nsel[0, 0]].tolist() == [0, 1, 2, 9, 15]


def test_budget_covering_sequence_keeps_all(oracle):
    lens = np.array([700, 64, 1], np.int32)
    scores = np.random.default_rng(0).standard_normal((3, 1, 11))
    idx, nsel = oracle.select_blocks(scores, lens, 64, 700, 64 * 11)
    assert idx[0, 0, :nsel[0, 0]].tolist() == list(range(11))
    assert idx[1, 0, :nsel[1, 0]].tolist() == [0]
    assert idx[2, 0, :nsel[2, 0]].tolist() == [0]


def test_empty_sequence(oracle):
    lens = np.array([0, 5], np.int32)
    scores = np.zeros((2, 1, 2))
    idx, nsel = oracle.select_blocks(scores, lens, 64, 128, 128)
    assert nsel.tolist() == [[0], [1]]
    assert idx[0, 0].tolist() == [-1, -1]


# ---------------------------------------------------------------- attention

def test_dense_equals_torch_sdpa(oracle):
    # With every block kept the method is plain softmax attention: compare
    # with torch's scaled_dot_product_attention in float64 (GQA by repeating
    # each KV head over its group).
    for seed, blk in ((0, 64), (1, 128)):
        wl, c = small_case(seed, blk=blk, budget=384)
        idx, nsel = W.identity_block_list(c["lens"], wl.num_kv_heads, blk, wl.nb_max)
        out, lse = oracle.attend(c["q"], c["k"], c["v"], c["lens"], idx, nsel, blk)
        q, K, V = (torch.from_numpy(widen(c[n])) for n in ("q", "k", "v"))
        G = wl.group
        for b in range(wl.batch):
            L = int(c["lens"][b])
            kk = K[b, :, :L].repeat_interleave(G, 0)
            vv = V[b, :, :L].repeat_interleave(G, 0)
            ref = torch.nn.functional.scaled_dot_product_attention(q[b][:, None], kk, vv)[:, 0]
            np.testing.assert_allclose(out[b], ref.numpy(), rtol=0, atol=1e-12)


def test_zero_keys_give_uniform_weights(oracle):
    # K = 0: every logit is 0, so lse = ln(number of valid kept tokens) and
    # out = the plain mean of the kept V rows.
    wl, c = small_case(3, lens=(300, 200))
    c["k"][:] = bits(np.zeros(1, np.float32))[0]
    kmax = 3
    idx = np.array([[[0, 2, 4], [1, 3, 4]], [[0, 3, -1], [2, 3, -1]]], np.int32)
    nsel = np.array([[3, 3], [2, 2]], np.int32)
    out, lse = oracle.attend(c["q"], c["k"], c["v"], c["lens"], idx, nsel, wl.block_size)
    V = widen(c["v"])
    G = wl.group
    for b in range(2):
        L = int(c["lens"][b])
        for h in range(2):
            toks = [t for j in idx[b, h, :nsel[b, h]] for t in range(j * 64, min(j * 64 + 64, L))]
            for g in range(G):
                assert abs(lse[b, h * G + g] - math.log(len(toks))) < 1e-12
                np.testing.assert_allclose(out[b, h * G + g], V[b, h, toks].mean(0), rtol=0, atol=1e-12)
    assert kmax == idx.shape[-1]


def test_constant_values_give_constant_output(oracle):
    wl, c = small_case(4)
    c["v"][:] = bits(np.array([1.5], np.float32))[0]
    kp = oracle.pool_project(c["k"], c["w_k"], c["lens"], wl.block_size)
    s = oracle.gate_scores(c["q"], c["w_q"], kp, c["lens"], wl.block_size, wl.max_seq_len)
    idx, nsel = oracle.select_blocks(s, c["lens"], wl.block_size, wl.max_seq_len, wl.budget_tokens)
    out, _ = oracle.attend(c["q"], c["k"], c["v"], c["lens"], idx, nsel, wl.block_size)
    np.testing.assert_allclose(out, 1.5, rtol=0, atol=1e-13)


def test_output_in_convex_hull_and_masking(oracle):
    # Output lies in the box spanned by the kept, valid V rows; tokens past
    # L_b are never read (NaN there must not leak).
    wl, c = small_case(5, lens=(300, 129))
    for b in range(2):
        L = int(c["lens"][b])
        c["k"][b, :, L:] = 0x7FC0
        c["v"][b, :, L:] = 0x7FC0                                   # bf16 NaN
    idx = np.array([[[1, 4], [0, 4]], [[0, 2], [1, 2]]], np.int32)
    nsel = np.full((2, 2), 2, np.int32)
    out, lse = oracle.attend(c["q"], c["k"], c["v"], c["lens"], idx, nsel, wl.block_size)
    assert np.isfinite(out).all() and np.isfinite(lse).all()
    V = widen(c["v"])
    G = wl.group
    for b in range(2):
        L = int(c["lens"][b])
        for h in range(2):
            toks = [t for j in idx[b, h] for t in range(j * 64, min(j * 64 + 64, L))]
            lo, hi = V[b, h, toks].min(0), V[b, h, toks].max(0)
            o = out[b, h * G:(h + 1) * G]
            assert (o >= lo - 1e-12).all() and (o <= hi + 1e-12).all()


def test_split_merge_invariance(oracle):
    # Attention over disjoint pieces of the kept list, merged by their
    # log-sum-exp, equals attention over the whole list (for 1, 2, 7 and
    # one-block-per-piece splits). This also pins lse: a wrong lse breaks the
    # merge.
    wl, c = small_case(6, Lmax=1024, lens=(1000, 777), budget=64 * 14)
    kp = oracle.pool_project(c["k"], c["w_k"], c["lens"], wl.block_size)
    s = oracle.gate_scores(c["q"], c["w_q"], kp, c["lens"], wl.block_size, wl.max_seq_len)
    idx, nsel = oracle.select_blocks(s, c["lens"], wl.block_size, wl.max_seq_len, wl.budget_tokens)
    full, full_lse = oracle.attend(c["q"], c["k"], c["v"], c["lens"], idx, nsel, wl.block_size)
    G = wl.group
    for S in (1, 2, 7, int(nsel.max())):
        parts_o, parts_l = [], []
        for p in range(S):
            sub = np.full_like(idx, -1)
            sub_n = np.zeros_like(nsel)
            for b in range(2):
                for h in range(2):
                    n = int(nsel[b, h])
                    lo, hi = p * n // S, (p + 1) * n // S
                    sub[b, h, :hi - lo] = idx[b, h, lo:hi]
                    sub_n[b, h] = hi - lo
            o, l = oracle.attend(c["q"], c["k"], c["v"], c["lens"], sub, sub_n, wl.block_size)
            parts_o.append(o)
            parts_l.append(l)
        for b in range(2):
            for hq in range(wl.num_q_heads):
                m, ml = oracle.merge(np.stack([po[b, hq] for po in parts_o]),
                                     np.array([pl[b, hq] for pl in parts_l]))
                np.testing.assert_allclose(m, full[b, hq], rtol=0, atol=1e-12)
                assert abs(ml - full_lse[b, hq]) < 1e-12
    assert G == 2


def test_block_order_does_not_matter(oracle):
    wl, c = small_case(7, Lmax=1024, lens=(1000, 1024), budget=64 * 9)
    idx = np.array([[[0, 3, 5, 8, 15], [1, 2, 9, 11, 15]], [[4, 6, 7, 10, 15], [0, 5, 12, 13, 15]]],
                   np.int32)
    nsel = np.full((2, 2), 5, np.int32)
    a, la = oracle.attend(c["q"], c["k"], c["v"], c["lens"], idx, nsel, wl.block_size)
    perm = idx[:, :, ::-1].copy()
    b_, lb = oracle.attend(c["q"], c["k"], c["v"], c["lens"], perm, nsel, wl.block_size)
    np.testing.assert_allclose(a, b_, rtol=0, atol=1e-13)
    np.testing.assert_allclose(la, lb, rtol=0, atol=1e-13)


def test_invalid_indices_are_skipped_and_empty_row(oracle):
    wl, c = small_case(8, lens=(300, 200))
    idx = np.array([[[0, 99, -3], [4, 1, 7]], [[-1, -1, -1], [3, 2, 0]]], np.int32)
    nsel = np.array([[3, 3], [3, 3]], np.int32)
    out, lse = oracle.attend(c["q"], c["k"], c["v"], c["lens"], idx, nsel, wl.block_size)
    ref, rlse = oracle.attend(c["q"], c["k"], c["v"], c["lens"],
                              np.array([[[0, -1, -1], [4, 1, -1]], [[-1, -1, -1], [3, 2, 0]]], np.int32),
                              np.array([[1, 2], [0, 3]], np.int32), wl.block_size)
    np.testing.assert_array_equal(out, ref)
    G = wl.group
    assert np.all(out[1, :G] == 0) and np.all(np.isneginf(lse[1, :G]))


def test_merge_all_empty(oracle):
    o, l = oracle.merge(np.ones((3, 4)), np.full(3, -np.inf))
    assert (o == 0).all() and l == -np.inf


def test_thread_count_reported(oracle):
    assert oracle.num_threads() >= 1


# ---------------------------------------------------------------- block-level ground truth

def test_block_mass_equals_torch_softmax_per_block(oracle):
    # The block mass is the dense softmax of each query head (torch float64)
    # summed over each block's valid tokens; lse is its log-denominator.
    for seed, blk in ((0, 64), (1, 128)):
        wl, c = small_case(seed, blk=blk)
        mass, lse = oracle.block_mass(c["q"], c["k"], c["lens"], blk)
        q, K = torch.from_numpy(widen(c["q"])), torch.from_numpy(widen(c["k"]))
        G, D = wl.group, wl.head_dim
        for b in range(wl.batch):
            L = int(c["lens"][b])
            NB = -(-L // blk)
            for h in range(wl.num_q_heads):
                z = (K[b, h // G, :L] @ q[b, h]) / math.sqrt(D)
                p = torch.softmax(z, 0)
                ref = torch.zeros(wl.nb_max, dtype=torch.float64)
                ref.index_add_(0, torch.arange(L) // blk, p)
                np.testing.assert_allclose(mass[b, h], ref.numpy(), rtol=0, atol=1e-13)
                assert abs(lse[b, h] - torch.logsumexp(z, 0).item()) < 1e-12
                assert np.all(mass[b, h, NB:] == 0.0)


def test_block_mass_zero_keys_is_token_share(oracle):
    # K = 0: uniform softmax, so block j holds n_j / L of the mass (the
    # partial last block its own token count) and lse = ln L.
    wl, c = small_case(5, lens=(300, 65))
    c["k"][:] = bits(np.zeros(1, np.float32))[0]
    mass, lse = oracle.block_mass(c["q"], c["k"], c["lens"], wl.block_size)
    for b, L in enumerate(int(x) for x in c["lens"]):
        n = [min(64, L - j * 64) for j in range(-(-L // 64))] + [0] * (wl.nb_max - (-(-L // 64)))
        for h in range(wl.num_q_heads):
            np.testing.assert_allclose(mass[b, h], np.array(n) / L, rtol=0, atol=1e-13)
            assert abs(lse[b, h] - math.log(L)) < 1e-12


def test_block_mass_constant_logit_per_block_closed_form(oracle):
    # K rows equal c_j * e_0 inside block j and q = e_0: every logit of block j
    # is c_j / sqrt(D), so mass_j = n_j exp(c_j / sqrt(D)) / sum_i n_i exp(c_i / sqrt(D)).
    wl, c = small_case(6, lens=(320, 200))
    D = wl.head_dim
    cj = np.array([2.0, -1.0, 0.5, 4.0, -3.0], np.float32)
    K = np.zeros((wl.batch, wl.num_kv_heads, wl.max_seq_len, D), np.float32)
    for j, v in enumerate(cj):
        K[:, :, j * 64:(j + 1) * 64, 0] = v
    Q = np.zeros((wl.batch, wl.num_q_heads, D), np.float32)
    Q[:, :, 0] = 1.0
    mass, lse = oracle.block_mass(bits(Q), bits(K), c["lens"], 64)
    for b, L in enumerate(int(x) for x in c["lens"]):
        NB = -(-L // 64)
        n = np.array([min(64, L - j * 64) for j in range(NB)], np.float64)
        w = n * np.exp(cj[:NB].astype(np.float64) / math.sqrt(D))
        for h in range(wl.num_q_heads):
            np.testing.assert_allclose(mass[b, h, :NB], w / w.sum(), rtol=1e-13, atol=0)
            assert abs(lse[b, h] - math.log(w.sum())) < 1e-12


def test_block_mass_single_block_and_empty(oracle):
    wl, c = small_case(7, lens=(40, 0))
    mass, lse = oracle.block_mass(c["q"], c["k"], c["lens"], wl.block_size)
    assert np.all(np.abs(mass[0, :, 0] - 1.0) < 1e-13) and np.all(mass[0, :, 1:] == 0.0)
    assert np.all(mass[1] == 0.0) and np.all(lse[1] == -np.inf)


# ---------------------------------------------------------------- gate variants

def _per_head_scores_torch(wl, c, kp):
    # every head's score with torch float64 matmuls: (W_q q_h) . kpool_j / sqrt(dg)
    q = torch.from_numpy(widen(c["q"]))
    Wq = torch.from_numpy(c["w_q"].astype(np.float64))
    KP = torch.from_numpy(kp)
    G = wl.group
    out = torch.full((wl.batch, wl.num_q_heads, wl.nb_max), float("nan"), dtype=torch.float64)
    for b in range(wl.batch):
        NB = -(-int(c["lens"][b]) // wl.block_size)
        for h in range(wl.num_q_heads):
            qg = Wq[h // G] @ q[b, h]
            out[b, h, :NB] = (KP[b, h // G, :NB] @ qg) / math.sqrt(wl.gate_dim)
    return out


@pytest.mark.parametrize("agg", [0, 1, 2])
def test_gate_aggregations_match_torch(oracle, agg):
    for seed, dg in ((0, 64), (1, 32)):
        wl, c = small_case(seed, dg=dg, lens=(320, 150))
        kp = oracle.pool_project(c["k"], c["w_k"], c["lens"], wl.block_size)
        got = oracle.gate_scores_agg(c["q"], c["w_q"], kp, c["lens"], wl.block_size, wl.max_seq_len, agg)
        sh = _per_head_scores_torch(wl, c, kp)
        G = wl.group
        for b in range(wl.batch):
            NB = -(-int(c["lens"][b]) // wl.block_size)
            for kvh in range(wl.num_kv_heads):
                grp = sh[b, kvh * G:(kvh + 1) * G, :NB]
                ref = {0: grp.mean(0), 1: grp.max(0).values, 2: torch.softmax(grp, 1).mean(0)}[agg]
                np.testing.assert_allclose(got[b, kvh, :NB], ref.numpy(), rtol=1e-12, atol=1e-15)
                assert np.all(np.isnan(got[b, kvh, NB:]))
                if agg == 2:
                    assert abs(got[b, kvh, :NB].sum() - 1.0) < 1e-12


def test_gate_aggregations_agree_when_heads_agree(oracle):
    # identical query heads: max = mean, and the softmax-mean is the softmax of the mean gate
    wl, c = small_case(2)
    G = wl.group
    for b in range(wl.batch):
        for kvh in range(wl.num_kv_heads):
            c["q"][b, kvh * G:(kvh + 1) * G] = c["q"][b, kvh * G]
    kp = oracle.pool_project(c["k"], c["w_k"], c["lens"], wl.block_size)
    mean = oracle.gate_scores_agg(c["q"], c["w_q"], kp, c["lens"], wl.block_size, wl.max_seq_len, 0)
    mx = oracle.gate_scores_agg(c["q"], c["w_q"], kp, c["lens"], wl.block_size, wl.max_seq_len, 1)
    sm = oracle.gate_scores_agg(c["q"], c["w_q"], kp, c["lens"], wl.block_size, wl.max_seq_len, 2)
    np.testing.assert_allclose(mx, mean, rtol=0, atol=1e-15)
    for b in range(wl.batch):
        NB = -(-int(c["lens"][b]) // wl.block_size)
        for kvh in range(wl.num_kv_heads):
            ref = torch.softmax(torch.from_numpy(mean[b, kvh, :NB]), 0).numpy()
            np.testing.assert_allclose(sm[b, kvh, :NB], ref, rtol=1e-12, atol=0)


def test_threshold_selection_brute_force(oracle):
    rng = np.random.default_rng(8)
    B, Hkv, blk, Lmax = 3, 2, 64, 64 * 40
    lens = np.array([Lmax, 64 * 17 + 5, 64], np.int32)
    scores = np.round(rng.standard_normal((B, Hkv, 40)), 1)  # many exact ties, some at the threshold
    for budget, tau in ((64 * 8, 0.3), (64 * 8, -np.inf), (64 * 8, np.inf), (64 * 40, 0.0), (64 * 3, -0.5)):
        idx, nsel = oracle.select_threshold(scores, lens, blk, Lmax, budget, tau)
        kmax = budget // blk
        for b in range(B):
            NB = -(-int(lens[b]) // blk)
            kb = min(kmax, NB)
            for h in range(Hkv):
                cand = [j for j in range(NB - 1) if scores[b, h, j] >= tau]
                cand.sort(key=lambda j: (-scores[b, h, j], j))
                ref = sorted(cand[:kb - 1]) + [NB - 1]
                assert nsel[b, h] == len(ref)
                assert list(idx[b, h, :len(ref)]) == ref and np.all(idx[b, h, len(ref):] == -1)
    top_i, top_n = oracle.select_blocks(scores, lens, blk, Lmax, 64 * 8)
    thr_i, thr_n = oracle.select_threshold(scores, lens, blk, Lmax, 64 * 8, -np.inf)
    assert np.array_equal(top_i, thr_i) and np.array_equal(top_n, thr_n)


# ---------------------------------------------------------------- block-sparse prefill

def prefill_case(seed, B=2, Hq=4, Hkv=2, D=64, dg=64, blk=64, Lmax=320, lens=(320, 200)):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, Lmax, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Lmax, D, generator=g).to(torch.bfloat16)
    u16 = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    wq = (torch.randn(Hkv, dg, D, generator=g) / math.sqrt(D)).numpy()
    wk = (torch.randn(Hkv, dg, D, generator=g) / math.sqrt(D)).numpy()
    return dict(q=u16(q), k=u16(k), v=u16(v), w_q=wq, w_k=wk, lens=np.array(lens, np.int32), blk=blk, G=Hq // Hkv)


def test_prefill_gate_identity_weights_closed_form(oracle):
    # W = I: s[i, j] = mean_h(mean of q_h over block i) . mean(K over block j) / sqrt(D)
    c = prefill_case(0)
    D = c["q"].shape[-1]
    eye = np.broadcast_to(np.eye(D, dtype=np.float32), (2, D, D)).copy()
    kp = oracle.pool_project(c["k"], eye, c["lens"], c["blk"])
    s = oracle.prefill_gate(c["q"], eye, kp, c["lens"], c["blk"])
    Q, K = widen(c["q"]), widen(c["k"])
    G, blk = c["G"], c["blk"]
    for b, L in enumerate(int(x) for x in c["lens"]):
        NB = -(-L // blk)
        for kvh in range(2):
            for i in range(NB):
                qb = Q[b, kvh * G:(kvh + 1) * G, i * blk:min(i * blk + blk, L)].mean(1).mean(0)
                for j in range(NB):
                    kb = K[b, kvh, j * blk:min(j * blk + blk, L)].mean(0)
                    if j <= i:
                        assert abs(s[b, kvh, i, j] - qb @ kb / math.sqrt(D)) < 1e-12
                    else:
                        assert math.isnan(s[b, kvh, i, j])
        assert np.all(np.isnan(s[b, :, NB:]))


def test_prefill_toy_gate_matches_hand_derivation(oracle):
    # Non-square, non-symmetric W_q (dg = 2, D = 4): a transposed or mis-strided
    # projection changes every score of this example.
    g = json.load(open(os.path.join(GOLDEN, "toy_prefill_gate.json")))
    dm = g["dims"]
    K = bits(np.array(g["K"], np.float32))[None, None]             # [1,1,6,4]
    q = bits(np.array(g["q"], np.float32))[None]                   # [1,2,6,4]
    wk = np.array(g["W_k"], np.float32)[None]
    wq = np.array(g["W_q"], np.float32)[None]
    lens = np.array([g["seq_len"]], np.int32)
    kp = oracle.pool_project(K, wk, lens, dm["block_size"])
    s = oracle.prefill_gate(q, wq, kp, lens, dm["block_size"])
    expect = np.array([[np.nan if x is None else x for x in row] for row in g["scores"]])
    np.testing.assert_allclose(s[0, 0], expect, rtol=0, atol=1e-13)  # NaN where j > i
    for budget, lists in g["selection"].items():
        idx, ns = oracle.prefill_select(s, lens, dm["block_size"], dm["max_seq_len"], int(budget))
        for i, want in enumerate(lists):
            assert list(idx[0, 0, i, :ns[0, 0, i]]) == want


def test_prefill_selection_is_decode_selection_per_query_block(oracle):
    c = prefill_case(1, Lmax=64 * 12, lens=(64 * 12, 64 * 7 + 3))
    kp = oracle.pool_project(c["k"], c["w_k"], c["lens"], c["blk"])
    s = oracle.prefill_gate(c["q"], c["w_q"], kp, c["lens"], c["blk"])
    s = np.round(s, 3)  # ties
    for budget in (64, 64 * 4, 64 * 20):
        idx, ns = oracle.prefill_select(s, c["lens"], 64, 64 * 12, budget)
        kmax = budget // 64
        for b, L in enumerate(int(x) for x in c["lens"]):
            NB = -(-L // 64)
            for i in range(12):
                if i >= NB:
                    assert ns[b, :, i].tolist() == [0, 0] and np.all(idx[b, :, i] == -1)
                    continue
                # the decode rule on a sequence of i + 1 blocks whose scores are row i
                row = np.full((2, 2, 12), np.nan)
                row[0, :, :i + 1] = s[b, :, i, :i + 1]
                r_idx, r_ns = oracle.select_blocks(row[:1], np.array([(i + 1) * 64], np.int32), 64, 64 * 12, budget)
                assert ns[b, :, i].tolist() == r_ns[0].tolist()
                assert np.array_equal(idx[b, :, i], r_idx[0]) and kmax == idx.shape[-1]


def test_prefill_dense_equals_torch_causal_sdpa(oracle):
    for blk in (64, 128):
        c = prefill_case(2, blk=blk, Lmax=256, lens=(256, 190))
        nbm = 256 // blk
        idx = np.full((2, 2, nbm, nbm), -1, np.int32)
        ns = np.zeros((2, 2, nbm), np.int32)
        for i in range(nbm):
            idx[:, :, i, :i + 1] = np.arange(i + 1)
            ns[:, :, i] = i + 1
        out, lse = oracle.prefill_attend(c["q"], c["k"], c["v"], c["lens"], idx, ns, blk)
        Q, K, V = (torch.from_numpy(widen(c[n])) for n in ("q", "k", "v"))
        for b, L in enumerate(int(x) for x in c["lens"]):
            kk = K[b, :, :L].repeat_interleave(c["G"], 0)
            vv = V[b, :, :L].repeat_interleave(c["G"], 0)
            ref = torch.nn.functional.scaled_dot_product_attention(Q[b, :, :L], kk, vv, is_causal=True)
            np.testing.assert_allclose(out[b, :, :L], ref.numpy(), rtol=0, atol=1e-12)
            z = (Q[b, :, :L] @ kk.transpose(1, 2)) / math.sqrt(Q.shape[-1])
            z = z.masked_fill(torch.triu(torch.ones(L, L, dtype=torch.bool), 1), float("-inf"))
            np.testing.assert_allclose(lse[b, :, :L], torch.logsumexp(z, -1).numpy(), rtol=0, atol=1e-12)
            assert np.all(out[b, :, L:] == 0.0) and np.all(lse[b, :, L:] == -np.inf)


def test_prefill_zero_keys_average_kept_causal_values(oracle):
    c = prefill_case(3, Lmax=64 * 5, lens=(64 * 5, 64 * 3 + 10))
    c["k"][:] = bits(np.zeros(1, np.float32))[0]
    idx = np.full((2, 2, 5, 2), -1, np.int32)
    ns = np.zeros((2, 2, 5), np.int32)
    for i in range(5):
        keep = [0, i] if i > 0 else [0]
        idx[:, :, i, :len(keep)] = keep
        ns[:, :, i] = len(keep)
    out, lse = oracle.prefill_attend(c["q"], c["k"], c["v"], c["lens"], idx, ns, 64)
    V = widen(c["v"])
    for b, L in enumerate(int(x) for x in c["lens"]):
        for h in range(4):
            for t in range(L):
                i = t // 64
                toks = [u for j in sorted(set([0, i])) for u in range(j * 64, j * 64 + 64) if u <= t]
                np.testing.assert_allclose(out[b, h, t], V[b, h // 2, toks].mean(0), rtol=0, atol=1e-12)
                assert abs(lse[b, h, t] - math.log(len(toks))) < 1e-12
