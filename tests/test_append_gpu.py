"""seer_append_kv: the step's new K/V rows land at position L_b - 1 of every
(b, kv head) row of both caches, bit for bit, and nothing else changes (rows
of empty sequences included). Then a fused step over the appended caches
equals one over caches written by hand."""
import numpy as np
import pytest
import torch

from block_sparse_attention_seer_b200 import api
from block_sparse_attention_seer_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("D,lens", [(128, [4096, 3001, 1, 0]), (64, [64, 65, 2048, 7])])
def test_append_writes_only_the_last_position(D, lens):
    wl = W.Workload("app", len(lens), 8, 2, D, 64, 64, 4096, 512)
    inp = W.make_inputs(wl, seed=3, device="cuda", seq_lens=np.array(lens, np.int32))
    dims = api.make_dims(**wl.dims())
    g = torch.Generator(device="cpu").manual_seed(9)
    k_new = torch.randn(wl.batch, wl.num_kv_heads, D, generator=g).to(torch.bfloat16).cuda()
    v_new = torch.randn(wl.batch, wl.num_kv_heads, D, generator=g).to(torch.bfloat16).cuda()
    k0, v0 = inp["k_cache"].clone(), inp["v_cache"].clone()
    api.seer_append_kv(dims, k_new, v_new, inp["seq_lens"], inp["k_cache"], inp["v_cache"])
    torch.cuda.synchronize()
    k_ref, v_ref = k0.clone(), v0.clone()
    for b, L in enumerate(lens):
        if L > 0:
            k_ref[b, :, L - 1] = k_new[b]
            v_ref[b, :, L - 1] = v_new[b]
    assert torch.equal(inp["k_cache"].view(torch.int16), k_ref.view(torch.int16))
    assert torch.equal(inp["v_cache"].view(torch.int16), v_ref.view(torch.int16))


def test_step_after_append_matches_hand_written_caches():
    wl = W.WORKLOADS["tiny"]
    inp = W.make_inputs(wl, seed=5, device="cuda")
    L = int(inp["seq_lens_host"][0])
    k_new = inp["k_cache"][:, :, L - 1].clone()
    v_new = inp["v_cache"][:, :, L - 1].clone()
    a = {k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    a["k_cache"][:, :, L - 1] = 0
    a["v_cache"][:, :, L - 1] = 0
    dims = api.make_dims(**wl.dims())
    api.seer_append_kv(dims, k_new, v_new, a["seq_lens"], a["k_cache"], a["v_cache"])
    outs = []
    for x in (inp, a):
        st = api.DecodeStep(**wl.dims(), budget_tokens=wl.budget_tokens)
        st.build_pool(x["k_cache"], x["w_k"], x["seq_lens"])
        st.fused_step(x["q"], x["k_cache"], x["v_cache"], x["w_q"], x["w_k"], x["seq_lens"])
        torch.cuda.synchronize()
        outs.append((st.out.clone(), st.block_idx.clone()))
    assert torch.equal(outs[0][1], outs[1][1])
    assert torch.equal(outs[0][0].view(torch.int16), outs[1][0].view(torch.int16))
