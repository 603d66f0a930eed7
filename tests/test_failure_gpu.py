"""Failure detection on the GPU without a fault: a bounded wait on a barrier
that nothing completes must give up within its limit, report it, and leave the
context usable; normal runs record no wait failure."""
import time

import numpy as np
import pytest
import torch

from block_sparse_attention_seer_b200 import api
from block_sparse_attention_seer_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_context_survives():
    t0 = time.perf_counter()
    assert api.seer_wait_selftest(20_000_000) == 1          # 20 ms limit, nothing arrives
    assert time.perf_counter() - t0 < 10.0
    # the context still works: a small decode step runs and is finite
    wl = W.WORKLOADS["tiny"]
    inp = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in W.make_inputs(wl, seed=1).items()}
    st = api.DecodeStep(**wl.dims(), budget_tokens=wl.budget_tokens)
    st.build_pool(inp["k_cache"], inp["w_k"], inp["seq_lens"])
    st.set_update_start(inp["seq_lens"])
    out, lse = st.step(inp["q"], inp["k_cache"], inp["v_cache"], inp["w_q"], inp["w_k"], inp["seq_lens"])
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


def test_no_wait_failures_in_normal_runs():
    api.seer_decode_wait_failures(reset=True)
    wl = W.WORKLOADS["decode_b16"].with_(batch=2)
    inp = W.make_inputs(wl, seed=2, device="cuda")
    st = api.DecodeStep(**wl.dims(), budget_tokens=wl.budget_tokens)
    st.build_pool(inp["k_cache"], inp["w_k"], inp["seq_lens"])
    st.set_update_start(inp["seq_lens"])
    for _ in range(3):
        st.step(inp["q"], inp["k_cache"], inp["v_cache"], inp["w_q"], inp["w_k"], inp["seq_lens"])
    torch.cuda.synchronize()
    assert api.seer_decode_wait_failures() == 0
    assert np.isfinite(st.out.float().cpu().numpy()).all()
