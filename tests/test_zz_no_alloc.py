"""dsa_layer_forward_static: the fused layer for callers that cannot allocate.

Serving engines that plan every device buffer up front (and forbid allocation
on the decode path), code running inside an allocator callback, or a runtime
given a fixed memory budget cannot pass the caller workspace that
dsa_layer_forward needs.  dsa_layer_forward_static takes that scratch from a
fixed 16 MiB array inside the library instead.  These tests call it through
the C ABI and check it against dsa_layer_forward with a caller workspace, on
two calls in a row (the array keeps the previous call's contents), and check
that a layer needing more scratch than the array holds is refused.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test; it also passes when run alone.
"""
import numpy as np
import pytest
import torch

import sparse_attention_sum_b200 as dsa
from sparse_attention_sum_b200 import runner
import workloads
from tests.gpu_common import assert_attend_close, dev, layer_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dsa.lib()
    yield
    assert dsa.get_device_status() == 0


def _static_call(dims, a, out, idx=None, lse=None):
    dsa.layer_forward_static(dims, a["q_idx"], a["k_idx"], a["w"], a["idx_scale"], a["q_pos"], a["kv_start"],
                             a["kv_len"], a["q"], a["k"], a["k_row_stride"], a["v"], a["v_row_stride"],
                             a["attn_scale"], out, lse=lse, idx_out=idx)


@pytest.mark.parametrize("name,sizes,top_k", [("decode", dict(B=4, S=5000), 2048),
                                              ("prefill", dict(T=300), 96),
                                              ("tiny", dict(), 16)])
def test_static_scratch_matches_caller_workspace(name, sizes, top_k):
    wl = workloads.make(name, **sizes)
    wl.top_k = top_k
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    ref = runner.dsa_layer(dims, **a, bufs=runner.LayerBuffers(dims, "cuda", t["q"].dtype, with_lse=True))
    torch.cuda.synchronize()
    for call in range(2):
        out = torch.full_like(ref.out, float("nan"))
        idx = torch.full_like(ref.idx, -7)
        lse = torch.full_like(ref.lse, float("nan"))
        _static_call(dims, a, out, idx, lse)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref.idx), f"call {call}: selection differs"
        assert_attend_close(out.double().cpu().numpy(), ref.out.double().cpu().numpy(), out.dtype,
                            f"{name} static call {call}")
        np.testing.assert_allclose(lse.cpu().numpy(), ref.lse.cpu().numpy(), atol=2e-3)


def test_static_scratch_keeps_selection_internal():
    wl = workloads.make("decode", B=2, S=3000)
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    ref = runner.dsa_layer(dims, **a)
    out = torch.empty_like(ref.out)
    _static_call(dims, a, out)           # no idx_out: the rows stay in the library's array
    torch.cuda.synchronize()
    assert_attend_close(out.double().cpu().numpy(), ref.out.double().cpu().numpy(), out.dtype, "no idx_out")


def test_static_scratch_refuses_layers_that_do_not_fit():
    wl = workloads.make("prefill", T=256)
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    big = dsa.Dims(**{**dims.as_dict(), "n_q": 4096, "n_kv": 4096})  # 64 MiB of scores
    with pytest.raises(dsa.DsaError) as ei:
        _static_call(big, a, torch.empty(1, device="cuda"))
    assert ei.value.name == "DSA_ERR_WORKSPACE"
    assert "16 MiB" in str(ei.value)
