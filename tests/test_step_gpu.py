"""The fused single-launch decode step (seer_decode_step) against the oracle
and against the separate five-call path.

* block lists: bit-exact with the oracle's (near-tie rows excluded) and
  bit-identical with seer_select_blocks' (same arithmetic, gate_core.cuh);
* refreshed pooled keys: identical to seer_kpool_update's;
* output: within the attention tolerance of the fp64 oracle given the same
  block list, and of the five-call path;
* repeated calls on one workspace give the same block lists and pooled keys
  bit for bit; with no more rows than SMs (each row split into fixed parts
  merged in a fixed order) the same outputs bit for bit too, with more rows
  (parts of rows taken dynamically, so the order in which partial results
  are combined varies) outputs within the rounding of the fp32 merge
  (REPEAT_TOL); the gate's row counters reset themselves, the launch counter
  grows by one grid per call and tags every row the call publishes.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_seer_b200 import api
from block_sparse_attention_seer_b200 import workloads as W
from oracle import oracle as O

from gpu_helpers import check_attention, check_indices, oracle_bits, to_dev

pytestmark = pytest.mark.gpu

# With more rows than SMs two calls on the same inputs may split a row's blocks
# differently among the CTAs (the decode takes work dynamically), so their bf16
# outputs may differ by the rounding of the fp32 merge: at most a bf16 unit in
# the last place or two.
REPEAT_TOL = 4e-3
REPEAT_LSE_TOL = 2e-5


def run_both(wl, inp):
    """Separate five-call step and fused step from the same pooled cache."""
    sep = api.DecodeStep(**wl.dims(), budget_tokens=wl.budget_tokens)
    sep.build_pool(inp["k_cache"], inp["w_k"], inp["seq_lens"])
    fus = api.DecodeStep(**wl.dims(), budget_tokens=wl.budget_tokens)
    fus.kpool.copy_(sep.kpool)
    sep.set_update_start(inp["seq_lens"])
    sep.step(inp["q"], inp["k_cache"], inp["v_cache"], inp["w_q"], inp["w_k"], inp["seq_lens"])
    fus.fused_step(inp["q"], inp["k_cache"], inp["v_cache"], inp["w_q"], inp["w_k"], inp["seq_lens"])
    torch.cuda.synchronize()
    return sep, fus


def check_step(wl, inp, batches=None):
    sep, fus = run_both(wl, inp)
    assert torch.equal(fus.block_idx, sep.block_idx)
    assert torch.equal(fus.num_selected, sep.num_selected)
    assert torch.equal(fus.kpool, sep.kpool)
    a = fus.out.float().cpu().numpy()
    b = sep.out.float().cpu().numpy()
    assert np.abs(a - b).max() <= 1e-2
    sel = slice(None) if batches is None else list(batches)
    c = oracle_bits(inp, batches)
    ora = O.step(c["q"], c["k"], c["v"], c["w_q"], c["w_k"], c["lens"], wl.block_size, wl.budget_tokens)
    gidx = fus.block_idx.cpu().numpy()[sel]
    gns = fus.num_selected.cpu().numpy()[sel]
    excluded = check_indices(gidx, gns, ora["block_idx"], ora["num_selected"], ora["scores"], c["lens"],
                             wl.block_size)
    o, l = O.attend(c["q"], c["k"], c["v"], c["lens"], gidx, gns, wl.block_size)
    mx, mean = check_attention(fus.out.cpu().double().numpy()[sel], fus.lse.cpu().double().numpy()[sel], o, l)
    return fus, excluded, mx, mean


@pytest.mark.parametrize("seed", range(5))
def test_fused_tiny(seed):
    wl = W.WORKLOADS["tiny"]
    check_step(wl, to_dev(W.make_inputs(wl, seed=seed)))


@pytest.mark.parametrize("shape", [
    (3, 32, 8, 128, 128, 64, 4096, [4096, 3001, 1], 1024),
    (2, 40, 8, 128, 128, 128, 8192, [8192, 5000], 1280),
    (2, 8, 1, 64, 128, 128, 2048, [2000, 129], 512),
    (4, 2, 2, 64, 64, 64, 1024, [64, 65, 127, 1000], 256),
    (2, 4, 2, 128, 64, 64, 3000, [2999, 1500], 640),
    (5, 8, 2, 128, 128, 64, 512, [0, 1, 64, 512, 300], 64),
    (5, 8, 2, 128, 128, 64, 512, [0, 1, 64, 512, 300], 4096),
    # 4 rows of up to 1024 blocks: 32 gate CTAs per row, but only 8 kept blocks -> 8 one-block parts, 8 slots
    (2, 8, 2, 128, 128, 64, 65536, [65536, 40001], 512),
])
def test_fused_small_shapes(shape):
    B, Hq, Hkv, D, dg, blk, Lmax, lens, budget = shape
    wl = W.Workload("fused", B, Hq, Hkv, D, dg, blk, Lmax, budget)
    check_step(wl, to_dev(W.make_inputs(wl, seed=12, pad_value=float("nan"), seq_lens=np.array(lens, np.int32))))


def test_fused_repeated_calls_reuse_workspace():
    wl = W.Workload("repeat", 3, 32, 8, 128, 128, 64, 4096, 1024)
    inp = to_dev(W.make_inputs(wl, seed=13, seq_lens=np.array([4096, 3001, 77], np.int32)))
    st = api.DecodeStep(**wl.dims(), budget_tokens=wl.budget_tokens)
    st.build_pool(inp["k_cache"], inp["w_k"], inp["seq_lens"])
    outs = []
    for _ in range(4):
        st.fused_step(inp["q"], inp["k_cache"], inp["v_cache"], inp["w_q"], inp["w_k"], inp["seq_lens"])
        torch.cuda.synchronize()
        outs.append((st.out.clone(), st.lse.clone(), st.block_idx.clone()))
    for o, l, i in outs[1:]:  # 24 rows: fixed parts, the same bits
        assert torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1]) and torch.equal(i, outs[0][2])
    ws = st.workspace()
    # the 64-bit launch counter grows by one grid (one CTA per SM) per call
    arrivals = int(ws[:8].view(torch.int64).item())
    assert arrivals == 4 * torch.cuda.get_device_properties(0).multi_processor_count
    assert api.seer_decode_wait_failures() == 0


def _state(st, rows):
    ws = st.workspace()
    off = (256 + rows * 4 + 255) // 256 * 256  # per-row decode states, 32 bytes each
    state = ws[off:off + rows * 32].view(torch.int32).view(rows, 8).cpu().numpy()
    return ws, state  # columns: ready epoch, slots handed out, front, back, positions counted in


def _three_calls(wl, inp, exact):
    st = api.DecodeStep(**wl.dims(), budget_tokens=wl.budget_tokens)
    st.build_pool(inp["k_cache"], inp["w_k"], inp["seq_lens"])
    outs = []
    for _ in range(3):
        st.fused_step(inp["q"], inp["k_cache"], inp["v_cache"], inp["w_q"], inp["w_k"], inp["seq_lens"])
        torch.cuda.synchronize()
        outs.append(st.out.clone())
    if exact:
        assert all(torch.equal(o, outs[0]) for o in outs[1:])
    else:
        assert all((o.float() - outs[0].float()).abs().max().item() <= REPEAT_TOL for o in outs[1:])
    return st


def test_fused_launch_epochs_rows_fit_the_grid():
    # 80 rows on a 148-SM part: each row is gated by one CTA, which then streams
    # the whole row and writes the output directly. Every call adds one grid (one
    # CTA per SM) to the launch counter and publishes every row with its epoch, so
    # nothing is reset between calls.
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rows = sms // 2 + 6
    wl = W.Workload("rows", rows // 2, 8, 2, 128, 128, 64, 1024, 256)
    lens = np.array([1024 - 7 * b for b in range(wl.batch)], np.int32)
    inp = to_dev(W.make_inputs(wl, seed=21, pad_value=float("nan"), seq_lens=lens))
    check_step(wl, inp)
    st = _three_calls(wl, inp, exact=True)
    ws, state = _state(st, rows)
    assert int(ws[:8].view(torch.int64).item()) == 3 * sms
    assert np.all(state[:, 0] == 3)  # published by the third call
    assert np.all(state[:, 4] == 0)  # one CTA per row: no partial slot was counted
    assert api.seer_decode_wait_failures() == 0


@pytest.mark.parametrize("case", ["tied_keys", "keep_all"])
def test_fused_one_row_per_cta_selection_without_threshold_pass(case):
    # 80 rows, one CTA each: the last warp waits for the selection's first threshold bin
    # to start the decode early. With every pooled key of a row equal (a constant K
    # along the sequence) the selection has no histogram pass (one key value: the
    # lowest indices), and with a budget above every row's length it keeps all
    # blocks without searching; either way the waiting warp must be released after
    # the selection, with nothing issued early.
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B = sms // 16 + 1  # x 8 heads: more than half the SMs, so one CTA per row
    Lmax = 2048
    budget = 512 if case == "tied_keys" else Lmax
    wl = W.Workload("noearly", B, 32, 8, 128, 128, 64, Lmax, budget)
    lens = np.array([Lmax - 50 * b for b in range(B)], np.int32)
    inp = W.make_inputs(wl, seed=23, seq_lens=lens)
    if case == "tied_keys":
        inp["k_cache"][:] = inp["k_cache"][:, :, :1, :]
    fus, _, _, _ = check_step(wl, to_dev(inp))
    if case == "keep_all":
        assert np.all(fus.num_selected.cpu().numpy() == (lens[:, None] + 63) // 64)
    assert api.seer_decode_wait_failures() == 0


def test_fused_rows_outnumber_the_grid_take_and_help():
    # More rows than SMs: CTAs take pieces of each row's list from the front and
    # help with the rows that have most left from the back. After three calls the
    # tally of fully taken rows (kept by launch parity) counts every row for the
    # third call and has been cleared for the fourth; every row's front met its back.
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B, Hkv = (sms + 40) // 4 + 1, 4
    rows = B * Hkv
    wl = W.Workload("many", B, 16, Hkv, 128, 128, 64, 2048, 512)
    lens = np.array([2048 - 37 * (b % 40) for b in range(B)], np.int32)
    inp = to_dev(W.make_inputs(wl, seed=22, pad_value=float("nan"), seq_lens=lens))
    check_step(wl, inp, batches=[0, 1, B - 1])
    st = _three_calls(wl, inp, exact=False)
    ws, state = _state(st, rows)
    assert int(ws[:8].view(torch.int64).item()) == 3 * sms
    tally = ws[8:16].view(torch.int32).cpu().numpy()  # by launch parity: epoch 3 counts in word 1
    assert tally[1] == rows and tally[0] == 0
    nsel = st.num_selected.view(-1).cpu().numpy()
    assert np.all(state[:, 0] == 3)
    assert np.all(state[:, 2] >= state[:, 3])                       # front met back: all taken
    assert np.all((state[:, 4] == nsel) | (state[:, 4] == 0))       # counted in fully, or one whole run
    assert api.seer_decode_wait_failures() == 0


@pytest.mark.parametrize("name,batches", [
    ("decode_b16", [0, 15]),
    ("large_block", [3]),
    ("ragged", [0, 63]),
    ("sweep_b1_keep10", None),
    ("sweep_b4_keep50", [2]),
])
def test_fused_full_size(name, batches):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, seed=0, device="cuda", pad_value=float("nan") if wl.ragged else None)
    _, excluded, mx, mean = check_step(wl, inp, batches)
    print(f"fused {name}: near-tie rows excluded {excluded}, out max {mx:.2e} mean {mean:.2e}")
