"""seer_decode_step_noalloc: the decode step for callers that cannot allocate.

Some callers cannot give the step a device workspace -- a plugin that its
host framework hands only input and output tensors, or a serving loop that
may not call cudaMalloc once it runs. This entry point keeps the step's
scratch in a static device array inside the library instead. Called through
the C ABI, two calls in a row must each reproduce the workspace entry point
(seer_decode_step) on the same inputs bit for bit: block lists, pooled keys,
outputs and lse (both shapes have no more rows than SMs, where the step
splits each row into fixed parts merged in a fixed order, so the same kernel
gives the same bits whichever scratch it uses). A second, different shape
runs in the same loop on the array the first left behind, so stale scratch
contents would show. Sizes whose scratch exceeds the array are refused with
SEER_ERR_UNSUPPORTED.

This file is collected last on purpose, and passes both alone in a fresh
process and after every other test (the array keeps the previous call's
contents; each call clears what must start at zero).
"""
import ctypes

import pytest
import torch

from block_sparse_attention_seer_b200 import api
from block_sparse_attention_seer_b200 import workloads as W

pytestmark = pytest.mark.gpu



def _outputs(wl, kpool0):
    dev = kpool0.device
    return dict(kpool=kpool0.clone(),
                block_idx=torch.zeros(wl.batch, wl.num_kv_heads, wl.kmax, dtype=torch.int32, device=dev),
                num_selected=torch.zeros(wl.batch, wl.num_kv_heads, dtype=torch.int32, device=dev),
                out=torch.zeros(wl.batch, wl.num_q_heads, wl.head_dim, dtype=torch.bfloat16, device=dev),
                lse=torch.zeros(wl.batch, wl.num_q_heads, dtype=torch.float32, device=dev))


def _call_noalloc(dims, inp, wl, o):
    return api.LIB.seer_decode_step_noalloc(
        ctypes.byref(dims), inp["q"].data_ptr(), inp["k_cache"].data_ptr(), inp["v_cache"].data_ptr(),
        inp["w_q"].data_ptr(), inp["w_k"].data_ptr(), inp["seq_lens"].data_ptr(), None, wl.budget_tokens, 0.0,
        o["kpool"].data_ptr(), o["block_idx"].data_ptr(), o["num_selected"].data_ptr(), o["out"].data_ptr(),
        o["lse"].data_ptr(), torch.cuda.current_stream().cuda_stream)


def _reference(name):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, seed=21, device="cuda")
    ref_st = api.DecodeStep(**wl.dims(), budget_tokens=wl.budget_tokens)
    ref_st.build_pool(inp["k_cache"], inp["w_k"], inp["seq_lens"])
    kpool0 = ref_st.kpool.clone()
    ref_st.fused_step(inp["q"], inp["k_cache"], inp["v_cache"], inp["w_q"], inp["w_k"], inp["seq_lens"])
    torch.cuda.synchronize()
    return wl, inp, api.make_dims(**wl.dims()), ref_st, kpool0


@pytest.mark.parametrize("names", [("decode_b16", "tiny"), ("tiny", "decode_b16")])
def test_noalloc_matches_workspace_entry_two_calls(names):
    cases = [_reference(n) for n in names]
    for _ in range(2):
        for wl, inp, dims, ref_st, kpool0 in cases:  # each shape on the array the other left
            o = _outputs(wl, kpool0)
            assert _call_noalloc(dims, inp, wl, o) == api.SEER_OK, api.LIB.seer_last_error_string().decode()
            torch.cuda.synchronize()
            assert torch.isfinite(o["out"].float()).all()
            assert torch.equal(o["out"], ref_st.out)
            assert torch.equal(o["lse"], ref_st.lse)
            assert torch.equal(o["block_idx"], ref_st.block_idx)
            assert torch.equal(o["num_selected"], ref_st.num_selected)
            assert torch.equal(o["kpool"], ref_st.kpool)


def test_noalloc_refuses_sizes_beyond_the_static_array():
    # 128 sequences x 32 heads of partial slots: above 32 MiB
    wl = W.WORKLOADS["ragged"].with_(batch=128)
    dims = api.make_dims(**wl.dims())
    assert api.seer_decode_step_workspace_size(dims, wl.budget_tokens) > (32 << 20)
    fake = torch.empty(256, dtype=torch.uint8, device="cuda")  # never read: refused before any launch
    p = fake.data_ptr()
    st = api.LIB.seer_decode_step_noalloc(ctypes.byref(dims), p, p, p, p, p, p, None, wl.budget_tokens, 0.0, p, p,
                                          p, p, None, None)
    assert st == api.SEER_ERR_UNSUPPORTED
    assert "static array" in api.LIB.seer_last_error_string().decode()
