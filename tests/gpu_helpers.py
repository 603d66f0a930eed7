"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same inputs, and compare with the stated tolerances.

Tolerances (fixed by the method's parity criteria):
  * block indices: bit-exact, except rows whose oracle gap between the worst
    kept and the best dropped non-last block is below 1e-6 (near ties);
  * attention output: max abs error <= 1e-2 and mean abs error <= 1e-3
    against the fp64 oracle, given the oracle's block list;
  * lse: abs error <= 1e-3 (fp32 softmax denominator);
  * kpool: rtol 1e-5 + atol 1e-6 (fp32 pooling and projection of bf16 data);
  * gate scores: abs error <= 1e-6, so that bit-exact selection is meaningful
    at the near-tie threshold.
"""
import numpy as np
import torch

from block_sparse_attention_seer_b200 import api
from block_sparse_attention_seer_b200 import workloads as W
from oracle import oracle as O

OUT_MAX_ABS = 1e-2
OUT_MEAN_ABS = 1e-3
LSE_ABS = 1e-3
SCORE_ABS = 1e-6
TIE_GAP = 1e-6


def to_dev(inp, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def gpu_step(inp, wl, num_splits=None):
    """Bulk pool build, then one decode step a1..a5 on the device; host copies of every output."""
    st = api.DecodeStep(**wl.dims(), budget_tokens=wl.budget_tokens, num_splits=num_splits)
    st.build_pool(inp["k_cache"], inp["w_k"], inp["seq_lens"])
    st.set_update_start(inp["seq_lens"])
    st.step(inp["q"], inp["k_cache"], inp["v_cache"], inp["w_q"], inp["w_k"], inp["seq_lens"])
    torch.cuda.synchronize()
    return st, dict(kpool=st.kpool.cpu().double().numpy(), scores=st.scores.cpu().double().numpy(),
                    block_idx=st.block_idx.cpu().numpy(), num_selected=st.num_selected.cpu().numpy(),
                    out=st.out.cpu().double().numpy(), lse=st.lse.cpu().double().numpy())


def gpu_attend(st, inp, block_idx, num_selected, num_splits=None):
    idx = torch.as_tensor(block_idx, dtype=torch.int32).cuda().contiguous()
    ns = torch.as_tensor(num_selected, dtype=torch.int32).cuda().contiguous()
    out, lse = st.attend(inp["q"], inp["k_cache"], inp["v_cache"], inp["seq_lens"], idx, ns, idx.shape[-1],
                         num_splits)
    torch.cuda.synchronize()
    return out.cpu().double().numpy(), lse.cpu().double().numpy()


def oracle_bits(inp, batches=None):
    """Oracle-form (uint16 bit) copies of the inputs, optionally for a subset of batch entries."""
    sl = slice(None) if batches is None else list(batches)

    def take(t):
        return W.bf16_bits(t[sl] if batches is not None else t)
    return dict(q=take(inp["q"]), k=take(inp["k_cache"]), v=take(inp["v_cache"]),
                w_q=inp["w_q"].cpu().numpy(), w_k=inp["w_k"].cpu().numpy(),
                lens=np.asarray(inp["seq_lens_host"])[sl].astype(np.int32))


def check_kpool(gpu_kp, ora_kp, lens, blk):
    for b in range(len(lens)):
        nb = -(-int(lens[b]) // blk)
        np.testing.assert_allclose(gpu_kp[b, :, :nb], ora_kp[b, :, :nb], rtol=1e-5, atol=1e-6)


def check_scores(gpu_s, ora_s, lens, blk):
    worst = 0.0
    for b in range(len(lens)):
        nb = -(-int(lens[b]) // blk)
        if nb == 0:
            continue
        err = np.abs(gpu_s[b, :, :nb] - ora_s[b, :, :nb]).max()
        worst = max(worst, float(err))
    assert worst <= SCORE_ABS, f"gate score error {worst:.3e} > {SCORE_ABS}"
    return worst


def check_indices(gpu_idx, gpu_n, ora_idx, ora_n, ora_scores, lens, blk):
    """Bit-exact block lists except near-tie rows; returns the number of rows excluded."""
    ties = O.near_tie_rows(ora_scores, ora_idx, ora_n, lens, blk, TIE_GAP)
    np.testing.assert_array_equal(gpu_n, ora_n)
    bad = []
    for b in range(gpu_idx.shape[0]):
        for h in range(gpu_idx.shape[1]):
            if ties[b, h]:
                continue
            if not np.array_equal(gpu_idx[b, h], ora_idx[b, h]):
                bad.append((b, h))
    assert not bad, f"block lists differ in rows {bad[:8]}"
    return int(ties.sum())


def check_attention(gpu_out, gpu_lse, ora_out, ora_lse):
    err = np.abs(gpu_out - ora_out)
    assert np.isfinite(gpu_out).all()
    assert err.max() <= OUT_MAX_ABS, f"max abs error {err.max():.3e}"
    assert err.mean() <= OUT_MEAN_ABS, f"mean abs error {err.mean():.3e}"
    finite = np.isfinite(ora_lse)
    assert (np.isfinite(gpu_lse) == finite).all()
    if finite.any():
        assert np.abs(gpu_lse[finite] - ora_lse[finite]).max() <= LSE_ABS
    return float(err.max()), float(err.mean())
