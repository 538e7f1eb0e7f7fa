"""GPU parity of the FP8 indexer (dsa_fp8_quantize, dsa_index_scores_fp8) against the oracle's FP8
reading: per-vector e4m3 codes with scale amax/448 (ik_llama.cpp PR #2063 ships the indexer tensors
in F8_E4M3), scores sum_h w * relu(scale * sq * sk * (q^ . k^)) (fak note, section 3)."""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
import sparse_attention_sum_b200 as dsa
from sparse_attention_sum_b200 import runner
import workloads
from tests.gpu_common import check_selection_in_band, dev, key_order, layer_inputs, report, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dsa.lib()
    dsa.set_kernel_policy(0)
    yield
    assert dsa.get_device_status() == 0


def _decode_codes(codes_u8: torch.Tensor) -> np.ndarray:
    """e4m3 bytes -> their values (torch's float8_e4m3fn decode, which the oracle's grid is pinned to)."""
    return codes_u8.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _quantize(x):
    codes = torch.empty(x.shape, dtype=torch.uint8, device="cuda")
    scales = torch.empty(x.shape[:-1], dtype=torch.float32, device="cuda")
    dsa.fp8_quantize(x, codes, scales)
    return codes, scales


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_codes_and_scales_equal_the_oracle(dtype):
    """Every code and scale, bit for bit: N(0,1) rows, rows spanning many binades (subnormal codes),
    a zero row, a row with one large entry, rows whose products land on e4m3 rounding midpoints."""
    g = torch.Generator().manual_seed(3)
    x = torch.randn(3000, 128, generator=g)
    x[1] = 0.0
    x[2] = torch.randn(128, generator=g) * 1e-3
    x[2, 5] = 40.0                                        # most codes subnormal
    x[3] = torch.logspace(-6, 3, 128)                     # every binade
    x[4] = torch.tensor(O.e4m3_grid()[1:][:64].tolist() * 2) * (1 - 2 * (torch.arange(128) % 2))
    mids = (O.e4m3_grid()[:-1] + O.e4m3_grid()[1:]) / 2  # exact midpoints, amax 448
    x[5, :120] = torch.tensor(mids[-120:])
    x[5, 120:] = 448.0
    x = x.to(dtype)
    xd = x.cuda()
    codes, scales = _quantize(xd)
    assert dsa.last_kernels() == ["fp8_quantize"]
    torch.cuda.synchronize()
    ref_codes, ref_scales = O.fp8_quantize(x)
    got = _decode_codes(codes)
    assert np.array_equal(got, ref_codes)
    assert np.array_equal(scales.cpu().numpy().astype(np.float64), ref_scales)
    assert np.all(got[1] == 0) and scales[1].item() == 1.0
    # a strided view (rows of a wider tensor) quantises the same
    wide = torch.zeros(3000, 192, dtype=dtype, device="cuda")
    wide[:, 32:160] = xd
    c2, s2 = _quantize(wide[:, 32:160])
    torch.cuda.synchronize()
    assert torch.equal(c2, codes) and torch.equal(s2, scales)


def _fp8_layer_scores(wl, t, dims, a):
    qc, qs = _quantize(a["q_idx"])
    kc, ks = _quantize(a["k_idx"])
    B, T, S = wl.batch, wl.n_q, wl.n_kv
    scores = torch.empty(B, T, S, dtype=torch.float32, device="cuda")
    dsa.index_scores_fp8(dims, qc, qs, kc, ks, a["w"], a["idx_scale"], a["q_pos"], a["kv_start"], a["kv_len"],
                         scores)
    assert dsa.last_kernels() == ["index_tc_fp8"]
    return scores


@pytest.mark.parametrize("name,sizes,top_k", [("prefill", dict(T=700), 256), ("decode", dict(B=3, S=5000), 2048)])
def test_fp8_indexer_is_exact_when_quantisation_is(name, sizes, top_k):
    """Integer indexer vectors whose largest magnitude is 7: the e4m3 scale is exactly 1/64 and the
    codes are 64*x, so the FP8 scores equal the plain scores exactly (oracle pinned), and the tcgen05
    kind::f8f6f4 kernel's fp32 accumulation of the code products is exact too: its scores and its
    selection must equal the oracle's bit for bit."""
    wl = workloads.make(name, exact_index="fp8", **sizes)
    wl.top_k = top_k
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    scores = _fp8_layer_scores(wl, t, dims, a)
    idx = torch.empty(wl.batch, wl.n_q, top_k, dtype=torch.int32, device="cuda")
    dsa.topk(dims, scores, a["q_pos"], a["kv_start"], a["kv_len"], top_k, idx)
    torch.cuda.synchronize()
    ref = O.index_scores(wl["q_idx"], wl["k_idx"], wl["w"], wl.idx_scale, wl["q_pos"], wl["kv_start"],
                         wl["kv_len"])
    got = scores.cpu().numpy().astype(np.float64)
    assert np.array_equal(got, ref)
    for b, tt in sample_rows(wl, 16):
        cand = O.visible_keys(int(wl["q_pos"][b, tt]), 0, wl.n_kv)
        ref8 = O.index_scores_fp8_row(wl["q_idx"][b, tt], wl["k_idx"][b][cand], wl["w"][b, tt], wl.idx_scale)
        assert np.array_equal(ref8, ref[b, tt, cand])
    assert np.array_equal(idx.cpu().numpy(), O.topk(ref, top_k, wl["q_pos"], wl["kv_start"], wl["kv_len"]))


@pytest.mark.parametrize("name,sizes,top_k,n_rows", [("prefill", dict(T=1000), 256, 64),
                                                     ("decode", dict(B=4, S=32768), 2048, 4),
                                                     ("chunked", dict(T=130, S=4500), 512, 40)])
def test_fp8_indexer_against_the_fp8_oracle(name, sizes, top_k, n_rows):
    """N(0,1) inputs (the benchmark recipe): the GPU quantises and scores; every sampled row's scores
    equal the FP8 oracle's within fp32 accumulation error (2e-5 of the row's score scale), the
    selection kernel is exact on the GPU's scores, and the selection sits inside the tie band of the
    FP8 oracle's scores.  Its recall against the bf16 selection is reported (a quality figure: e4m3
    noise, not a parity bar)."""
    wl = workloads.make(name, **sizes)
    wl.top_k = top_k
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    scores = _fp8_layer_scores(wl, t, dims, a)
    idx = torch.empty(wl.batch, wl.n_q, top_k, dtype=torch.int32, device="cuda")
    dsa.topk_set(dims, scores, a["q_pos"], a["kv_start"], a["kv_len"], top_k, idx)
    torch.cuda.synchronize()
    g_idx = idx.cpu().numpy()
    worst, recall, diffs = 0.0, [], 0
    for b, tt in sample_rows(wl, n_rows):
        cand = O.visible_keys(int(wl["q_pos"][b, tt]), int(wl["kv_start"][b]), int(wl["kv_len"][b]))
        ref8 = O.index_scores_fp8_row(wl["q_idx"][b, tt], wl["k_idx"][b][cand], wl["w"][b, tt], wl.idx_scale)
        gs = scores[b, tt].cpu().numpy().astype(np.float64)
        assert np.all(np.isneginf(np.delete(gs, cand)))
        err = np.abs(gs[cand] - ref8).max() / max(1.0, np.abs(ref8).max())
        worst = max(worst, err)
        assert err <= 2e-5, (b, tt, err)
        assert g_idx[b, tt].tolist() == key_order(O.topk_row(cand, gs[cand], top_k).tolist())
        diffs += check_selection_in_band(g_idx[b, tt], cand, ref8, top_k, f"fp8 {name} {(b, tt)}") > 0
        ref16 = O.index_scores_row(wl["q_idx"][b, tt], wl["k_idx"][b][cand], wl["w"][b, tt], wl.idx_scale)
        k = min(top_k, cand.size)
        recall.append(len(set(O.topk_row(cand, ref16, k).tolist()) & set(g_idx[b, tt, :k].tolist())) / k)
    report(f"fp8 indexer {name}", rows=n_rows, score_err_over_scale=f"{worst:.2e}", rows_in_tie_band=diffs,
           recall_vs_bf16_min=f"{min(recall):.4f}", recall_vs_bf16_mean=f"{np.mean(recall):.4f}")


def test_fp8_layer_chain_attends_over_the_fp8_selection():
    """runner.dsa_layer_fp8 (quantise queries, FP8 scores, top-k set, attend) gives the same output as the
    three calls made by hand, and launches exactly those kernels."""
    wl = workloads.make("prefill", T=300)
    wl.top_k = 96
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    kc, ks = _quantize(a["k_idx"])
    bufs = runner.dsa_layer_fp8(dims, k_codes=kc, k_scales=ks, **a)
    assert dsa.last_kernels() == ["attend_tc"]
    scores = _fp8_layer_scores(wl, t, dims, a)
    idx = torch.empty_like(bufs.idx)
    dsa.topk_set(dims, scores, a["q_pos"], a["kv_start"], a["kv_len"], wl.top_k, idx)
    out = torch.empty_like(bufs.out)
    dsa.sparse_attend(dims, a["q"], a["k"], a["k_row_stride"], a["v"], a["v_row_stride"], idx, wl.top_k,
                      a["attn_scale"], out)
    torch.cuda.synchronize()
    assert torch.equal(idx, bufs.idx)
    assert torch.equal(out, bufs.out)


@pytest.mark.parametrize("sizes", [dict(B=5, S=32768), dict(B=2, S=70000), dict(B=3, S=5000)])
def test_fused_fp8_index_topk_equals_fp8_scores_then_topk_set(sizes):
    """dsa_index_topk_fp8 (a cluster per query row, FP8 scores kept in shared memory) selects exactly what
    dsa_index_scores_fp8 + dsa_topk_set select: one query per row uses the same tcgen05 tile shape, so
    the scores agree bit for bit and so does the selection."""
    wl = workloads.make("decode", **sizes)
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    qc, qs = _quantize(a["q_idx"])
    kc, ks = _quantize(a["k_idx"])
    fused = torch.full((wl.batch, 1, wl.top_k), 12345, dtype=torch.int32, device="cuda")
    dsa.index_topk_fp8(dims, qc, qs, kc, ks, a["w"], a["idx_scale"], a["q_pos"], a["kv_start"], a["kv_len"],
                       wl.top_k, fused)
    assert dsa.last_kernels() == ["index_topk_fp8"]
    scores = torch.empty(wl.batch, 1, wl.n_kv, dtype=torch.float32, device="cuda")
    dsa.index_scores_fp8(dims, qc, qs, kc, ks, a["w"], a["idx_scale"], a["q_pos"], a["kv_start"], a["kv_len"],
                         scores)
    ref = torch.empty_like(fused)
    dsa.topk_set(dims, scores, a["q_pos"], a["kv_start"], a["kv_len"], wl.top_k, ref)
    torch.cuda.synchronize()
    assert torch.equal(fused, ref)
