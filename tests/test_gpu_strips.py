"""Balanced causal strips on one GPU: the strips of a prefill, run one after another through the C ABI,
give exactly the rows of the whole layer (attention outputs, selections and log-sum-exps).  A row's scores,
selection and attention depend only on its own query and the keys it sees, in a fixed order, so the split
changes no bit."""
import numpy as np
import pytest
import torch

import workloads
from sparse_attention_sum_b200 import runner
from sparse_attention_sum_b200 import strips as S
from gpu_common import dev, layer_inputs


@pytest.mark.gpu
@pytest.mark.parametrize("T,world", [(1000, 3), (4096, 4)])
def test_strips_reproduce_the_whole_layer(T, world):
    wl = workloads.make("prefill", T=T)
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    full = runner.LayerBuffers(dims, "cuda", t["q"].dtype, with_idx=True, with_lse=True)
    runner.dsa_layer(dims, **a, bufs=full)
    torch.cuda.synchronize()
    plan = S.causal_strips(wl["q_pos"][0].numpy(), world, wl.top_k, kv_start=int(wl["kv_start"][0]),
                           n_keys=wl.n_kv)
    assert plan[-1].b == T and all(s.b > s.a for s in plan)
    for s in plan:
        got = S.run_strip(t, s, wl.vd, wl.top_k, wl.idx_scale, wl.attn_scale)
        torch.cuda.synchronize()
        assert torch.equal(got.idx[0], full.idx[0, s.a:s.b]), s
        assert torch.equal(got.out[0], full.out[0, s.a:s.b]), s
        assert torch.equal(got.lse[0], full.lse[0, s.a:s.b]), s
