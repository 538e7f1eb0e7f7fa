"""GPU parity: every stage of the CUDA path against the CPU oracle (needs a B200).

Small cases compare every element; full-size workloads (in the launch
configuration bench.py times) compare sampled rows element by element and
check structural properties on every row.
"""

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
import sparse_attention_sum_b200 as dsa
from sparse_attention_sum_b200 import runner
import workloads
from tests.gpu_common import (ATOL, assert_attend_close, check_selection_in_band, cosine, dev, key_order,
                              kv_views, layer_inputs, report, sample_rows)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dsa.lib()  # fail loudly if the library is missing
    dsa.set_kernel_policy(0)
    yield
    assert dsa.get_device_status() == 0


def _np(t):
    return t.detach().to(torch.float64).cpu().numpy()


def _run_stages(wl, t):
    """Index scores, top-k and attend as three separate C-ABI calls."""
    dims, a = layer_inputs(wl, t)
    B, T, S = wl.batch, wl.n_q, wl.n_kv
    scores = torch.empty(B, T, S, dtype=torch.float32, device="cuda")
    dsa.index_scores(dims, a["q_idx"], a["k_idx"], a["w"], a["idx_scale"], a["q_pos"], a["kv_start"],
                     a["kv_len"], scores)
    idx = torch.empty(B, T, wl.top_k, dtype=torch.int32, device="cuda")
    vals = torch.empty(B, T, wl.top_k, dtype=torch.float32, device="cuda")
    dsa.topk(dims, scores, a["q_pos"], a["kv_start"], a["kv_len"], wl.top_k, idx, vals)
    out = torch.empty(B, T, wl.heads, wl.vd, dtype=t["q"].dtype, device="cuda")
    lse = torch.empty(B, T, wl.heads, dtype=torch.float32, device="cuda")
    dsa.sparse_attend(dims, a["q"], a["k"], a["k_row_stride"], a["v"], a["v_row_stride"], idx, wl.top_k,
                      a["attn_scale"], out, lse)
    torch.cuda.synchronize()
    return dims, a, scores, idx, vals, out, lse


# ------------------------------------------------------------- tiny (fp32)
def test_tiny_layer_is_exact_against_oracle():
    wl = workloads.make("tiny")
    t = dev(wl)
    dims, a, scores, idx, vals, out, lse = _run_stages(wl, t)
    ref_scores = O.index_scores(wl["q_idx"], wl["k_idx"], wl["w"], wl.idx_scale, wl["q_pos"],
                                wl["kv_start"], wl["kv_len"])
    got = _np(scores)
    # integer inputs, power-of-two scale and weights: exact scores, bit-identical selection
    assert np.array_equal(got, ref_scores)
    ref_idx = O.topk(ref_scores, wl.top_k, wl["q_pos"], wl["kv_start"], wl["kv_len"])
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    gv = vals.cpu().numpy()
    for tt in range(wl.n_q):
        n = min(wl.top_k, tt + 1)
        assert np.array_equal(gv[0, tt, :n], ref_scores[0, tt, ref_idx[0, tt, :n]])
        assert np.all(np.isneginf(gv[0, tt, n:]))
    # attention over the (identical) selection: fp32 tolerance
    K, V = kv_views(wl)
    ref_out, ref_lse = O.sparse_attend(wl["q"], K, V, ref_idx, wl.attn_scale)
    assert_attend_close(_np(out), ref_out, torch.float32, "tiny attend")
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=1e-4)
    # the fused call: dsa_topk's set listed in key order, attended as in the composition
    bufs = runner.dsa_layer(dims, **a)
    torch.cuda.synchronize()
    assert torch.equal(bufs.idx, key_order(idx))
    again = torch.empty_like(out)
    dsa.sparse_attend(dims, a["q"], a["k"], a["k_row_stride"], a["v"], a["v_row_stride"], bufs.idx, wl.top_k,
                      a["attn_scale"], again)
    torch.cuda.synchronize()
    assert torch.equal(bufs.out, again)
    assert_attend_close(_np(bufs.out), ref_out, torch.float32, "tiny fused layer")


def test_tiny_layer_covering_all_keys_is_dense_attention():
    wl = workloads.make("tiny")
    wl.top_k = 64
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    bufs = runner.dsa_layer(dims, **a)
    torch.cuda.synchronize()
    K, V = kv_views(wl)
    dense = O.dense_causal_attend(wl["q"], K, V, wl.attn_scale, wl["q_pos"], wl["kv_start"], wl["kv_len"])
    assert_attend_close(_np(bufs.out), dense, torch.float32, "dense reduction")


# --------------------------------- tensor-core indexer on exact (integer) scores
@pytest.mark.parametrize("name,sizes,top_k", [("prefill", dict(T=1000), 256), ("decode", dict(B=3, S=5000), 2048),
                                              ("chunked", dict(T=130, S=4500), 512)])
def test_integer_indexer_on_tensor_cores_is_exact(name, sizes, top_k):
    """The bf16 indexer at its full shape (64 heads x 128) on integer inputs (q_I, k_I in [-4, 4],
    w in {1/2, 1, 2, 4}, scale 1/8): every score is a multiple of 1/16 below 2^17, so the tcgen05
    kernel's TMEM accumulation, relu*w epilogue, signed-zero rule and skipped tiles must give the
    oracle's scores exactly, and the selection must be the oracle's bit for bit (with many genuine
    ties for the index tie-break).  Prefill runs 8 query tiles x 8 key tiles with ragged tails,
    decode the narrow two-CTA-per-SM configuration with key-range splits, chunked a causal offset
    with hot spots."""
    wl = workloads.make(name, exact_index=True, **sizes)
    wl.top_k = top_k
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    B, T, S = wl.batch, wl.n_q, wl.n_kv
    scores = torch.empty(B, T, S, dtype=torch.float32, device="cuda")
    dsa.index_scores(dims, a["q_idx"], a["k_idx"], a["w"], a["idx_scale"], a["q_pos"], a["kv_start"],
                     a["kv_len"], scores)
    assert dsa.last_kernels() == ["index_tc"]
    idx = torch.empty(B, T, top_k, dtype=torch.int32, device="cuda")
    dsa.topk(dims, scores, a["q_pos"], a["kv_start"], a["kv_len"], top_k, idx)
    fused = runner.dsa_layer(dims, **a)
    assert dsa.last_kernels() == (["index_topk", "attend_tc"] if T == 1 else ["index_tc", "topk_set", "attend_tc"])
    torch.cuda.synchronize()
    ref = O.index_scores(wl["q_idx"], wl["k_idx"], wl["w"], wl.idx_scale, wl["q_pos"], wl["kv_start"],
                         wl["kv_len"])
    got = scores.cpu().numpy().astype(np.float64)
    assert np.array_equal(got, ref)
    assert not np.any(np.signbit(got[got == 0]))                  # zero scores are +0
    ref_idx = O.topk(ref, top_k, wl["q_pos"], wl["kv_start"], wl["kv_len"])
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert torch.equal(fused.idx, key_order(torch.tensor(ref_idx, dtype=torch.int32, device="cuda")))
    n_ties = int(sum(np.sum(ref[b, tt] == ref[b, tt, ref_idx[b, tt, -1]]) > 1
                     for b in range(B) for tt in range(T) if ref_idx[b, tt, -1] >= 0))
    report(f"exact indexer {name}", rows=B * T, rows_with_tie_at_kth=n_ties)


# --------------------------------------------------------- top-k edge cases
def _topk_case(scores_np, q_pos, kv_start, kv_len, k, kpool=0):
    B, T, S = scores_np.shape
    d = dsa.Dims(batch=B, n_q=T, n_kv=S, kpool=kpool, top_k=k)
    sc = torch.tensor(scores_np, dtype=torch.float32, device="cuda")
    qp = torch.tensor(q_pos, dtype=torch.int32, device="cuda")
    ks = torch.tensor(kv_start, dtype=torch.int32, device="cuda")
    kl = torch.tensor(kv_len, dtype=torch.int32, device="cuda")
    idx = torch.full((B, T, k), 12345, dtype=torch.int32, device="cuda")
    vals = torch.empty(B, T, k, dtype=torch.float32, device="cuda")
    dsa.topk(d, sc, qp, ks, kl, k, idx, vals)
    set_idx = torch.full_like(idx, 12345)
    set_vals = torch.empty_like(vals)
    dsa.topk_set(d, sc, qp, ks, kl, k, set_idx, set_vals)
    torch.cuda.synchronize()
    got = idx.cpu().numpy()
    # the set form: the same keys in ascending key order, each with its score
    assert torch.equal(set_idx, key_order(idx))
    gv, sv = vals.cpu().numpy(), set_vals.cpu().numpy()
    for b in range(B):
        for t in range(T):
            pos = {int(x): i for i, x in enumerate(got[b, t]) if x >= 0}
            for j, x in enumerate(set_idx[b, t].tolist()):
                assert (sv[b, t, j] == gv[b, t, pos[x]]) if x >= 0 else np.isneginf(sv[b, t, j])
    for b in range(B):
        for t in range(T):
            if kpool:
                npools = O.n_pools_of(kv_start[b], kv_len[b], kpool)
                cand = O.visible_pools(q_pos[b][t], kv_start[b], min(npools, S), kpool)
            else:
                cand = O.visible_keys(q_pos[b][t], kv_start[b], min(kv_len[b], S))
            want = O.topk_row(cand, scores_np[b, t, cand].astype(np.float64), k)
            assert got[b, t].tolist() == want.tolist(), (b, t, k)
    return got


@pytest.mark.parametrize("S,k", [(1, 1), (7, 16), (64, 16), (300, 37), (4096, 2048), (5000, 4096),
                                 (33000, 2048), (50000, 2048), (2049, 2048)])
def test_topk_bit_exact_with_heavy_ties(S, k):
    rng = np.random.default_rng(S + k)
    T = 6
    # integer-valued scores: many exact ties exercise the index tie-break
    scores = rng.integers(-3, 4, size=(2, T, S)).astype(np.float32) * 0.5
    scores[0, 0, :] = 0.0                             # an all-equal row
    scores[1, 1, ::2] = -0.0                          # signed zeros equal +0
    q_pos = [[S - 1, S // 2, 0, S - 1, 3, S + 5], [S - 1, S - 1, S // 3, 1, S - 2, 2 * S]]
    kv_start = [0, min(2, S - 1)]
    kv_len = [S, max(1, S - 3)]
    _topk_case(scores, q_pos, kv_start, kv_len, k)


def test_topk_long_rows_with_adversarial_structure():
    # rows of 32768 keys (the 1024-thread kernel) built against estimates of the threshold from a
    # regular subset of the row: row 0 puts the top k at positions 0 and 1 mod 32 (a comb), row 1 makes
    # every key at 16 mod 32 large, row 2 is plain normal data, row 3 has 3000 keys tied at the k-th
    # largest value; each set of rows is also seen from an unaligned first visible key.  All exact
    # against the oracle.
    rng = np.random.default_rng(7)
    S, k, T = 32768, 2048, 4
    scores = rng.standard_normal((1, T, S)).astype(np.float32)
    pos = np.arange(S)
    comb = (pos % 32 == 0) | (pos % 32 == 1)
    scores[0, 0, comb] = 10.0 + rng.random(int(comb.sum())).astype(np.float32)
    strided = pos % 32 == 16
    scores[0, 1, strided] = 10.0 + rng.random(int(strided.sum())).astype(np.float32)
    kth = np.sort(scores[0, 3])[::-1][k - 1]
    tie = rng.choice(S, 3000, replace=False)
    scores[0, 3, tie] = kth
    q_pos = [[S - 1] * T]
    for start in (0, 5, 3):
        _topk_case(scores, q_pos, [start], [S], k)


def test_topk_distinct_and_padded_rows():
    rng = np.random.default_rng(0)
    S = 9000
    scores = rng.standard_normal((3, 4, S)).astype(np.float32)
    q_pos = [[S - 1, 100, 5, 2047], [4, 3, S - 1, 2500], [S - 1, S - 1, S - 1, S - 1]]
    kv_start = [0, 5, 1000]      # batch 1 row 1: padded query (q_pos < kv_start)
    kv_len = [S, S, 6000]
    got = _topk_case(scores, q_pos, kv_start, kv_len, 2048)
    assert np.all(got[1, 1] == O.INVALID)


def test_topk_pool_mode_visibility():
    rng = np.random.default_rng(1)
    P = 300
    scores = rng.integers(-2, 3, size=(2, 5, P)).astype(np.float32)
    q_pos = [[2, 3, 7, 1199, 600], [16, 17, 20, 1199, 100]]
    _topk_case(scores, q_pos, [0, 17], [1200, 1200], 64, kpool=4)


# -------------------------------------------------------- attend edge cases
@pytest.mark.parametrize("dtype,H,Hk,kd,vd", [(torch.float32, 4, 4, 32, 24), (torch.float32, 8, 2, 40, 40),
                                              (torch.bfloat16, 128, 1, 576, 512),
                                              (torch.bfloat16, 64, 1, 512, 512),
                                              (torch.bfloat16, 3, 1, 70, 33)])
def test_attend_set_semantics(dtype, H, Hk, kd, vd):
    rng = np.random.default_rng(H + kd)
    B, T, S, W = 2, 5, 300, 40
    shared = Hk == 1 and kd >= vd
    q = torch.tensor(rng.standard_normal((B, T, H, kd)), dtype=dtype)
    if shared:
        lat = torch.tensor(rng.standard_normal((B, S, kd)) * 0.5, dtype=dtype)
        K, V = lat.unsqueeze(2), lat[..., :vd].unsqueeze(2)
        k_dev, v_dev, ks, vs = lat.cuda(), lat.cuda(), kd, kd
    else:
        K = torch.tensor(rng.standard_normal((B, S, Hk, kd)), dtype=dtype)
        V = torch.tensor(rng.standard_normal((B, S, Hk, vd)), dtype=dtype)
        k_dev, v_dev, ks, vs = K.cuda(), V.cuda(), Hk * kd, Hk * vd
    idx = rng.integers(-1, S, size=(B, T, W)).astype(np.int32)
    idx[0, 0, :] = -1                     # empty row
    idx[0, 1, :] = 7                      # one key repeated
    idx[0, 2, ::3] = S + 11               # out of range
    idx[1, 0, :] = np.arange(W) % 5       # duplicates of five keys
    idx[1, 1, :] = rng.permutation(S)[:W]
    d = dsa.Dims(batch=B, n_q=T, n_kv=S, heads=H, kv_heads=Hk, kd=kd, vd=vd, top_k=W,
                 dtype=dsa.F32 if dtype == torch.float32 else dsa.BF16)
    out = torch.empty(B, T, H, vd, dtype=dtype, device="cuda")
    lse = torch.empty(B, T, H, dtype=torch.float32, device="cuda")
    dsa.sparse_attend(d, q.cuda(), k_dev, ks, v_dev, vs, torch.tensor(idx).cuda(), W, 0.3, out, lse)
    torch.cuda.synchronize()
    ref, ref_lse = O.sparse_attend(q, K, V, idx, 0.3)
    assert_attend_close(_np(out), ref, dtype, f"attend {dtype} H{H} kd{kd}")
    g_lse = lse.cpu().numpy()
    assert np.all(np.isneginf(g_lse[0, 0])) and np.all(_np(out)[0, 0] == 0)
    fin = np.isfinite(ref_lse)
    np.testing.assert_allclose(g_lse[fin], ref_lse[fin], atol=2e-3 if dtype == torch.bfloat16 else 1e-4)


# -------------------------------------------------- bf16 MLA layer (small)
@pytest.mark.parametrize("name,sizes", [("prefill", dict(T=333)), ("decode", dict(B=3, S=5000)),
                                        ("chunked", dict(T=130, S=4500))])
def test_small_bf16_layer_against_oracle(name, sizes):
    wl = workloads.make(name, **sizes)
    if name == "prefill":
        wl.top_k = 128
    t = dev(wl)
    dims, a, scores, idx, vals, out, lse = _run_stages(wl, t)
    g_scores = scores.cpu().numpy().astype(np.float64)
    g_idx = idx.cpu().numpy()
    K, V = kv_views(wl)
    B, T = wl.batch, wl.n_q
    rows = [(b, tt) for b in range(B) for tt in range(T)] if B * T <= 400 else sample_rows(wl, 40)
    n_diff_rows = 0
    for b, tt in rows:
        p, ks, kl = int(wl["q_pos"][b, tt]), int(wl["kv_start"][b]), int(wl["kv_len"][b])
        cand = O.visible_keys(p, ks, kl)
        ref = O.index_scores_row(wl["q_idx"][b, tt], wl["k_idx"][b][cand], wl["w"][b, tt], wl.idx_scale)
        gs = g_scores[b, tt, cand]
        scale_ = max(1.0, np.abs(ref).max())
        assert np.abs(gs - ref).max() <= 2e-5 * scale_, (b, tt, np.abs(gs - ref).max())
        invis = np.ones(wl.n_kv, bool)
        invis[cand] = False
        assert np.all(np.isneginf(g_scores[b, tt, invis]))
        # selection kernel alone: bit-exact against the oracle top-k of the GPU's own scores
        assert g_idx[b, tt].tolist() == O.topk_row(cand, gs, wl.top_k).tolist()
        # end to end: inside the tie band of the oracle's scores
        n_diff_rows += check_selection_in_band(g_idx[b, tt], cand, ref, wl.top_k, f"{name} row {(b, tt)}") > 0
        # attend over the GPU's own selection
        ro, rl = O.sparse_attend_row(wl["q"][b, tt], K[b], V[b], g_idx[b, tt], wl.attn_scale)
        assert_attend_close(_np(out[b, tt]), ro, torch.bfloat16, f"{name} attend {(b, tt)}")
    assert n_diff_rows <= max(1, len(rows) // 10)
    # the fused layer lists the same selection in key order; its attention matches the composition
    fused = runner.dsa_layer(dims, **a)
    torch.cuda.synchronize()
    assert torch.equal(fused.idx, key_order(idx))
    assert_attend_close(_np(fused.out), _np(out), torch.bfloat16, f"{name} fused vs composition", gpu_pair=True)


@pytest.mark.parametrize("name,sizes,top_k", [("prefill", dict(T=300), 96), ("decode", dict(B=2, S=5000), 2048)])
def test_fused_layer_all_scores_tied_takes_lowest_keys(name, sizes, top_k):
    # indexer weights 0: every visible score is 0, so the tie rule alone decides
    wl = workloads.make(name, **sizes)
    wl.top_k = top_k
    t = dev(wl)
    t["w"].zero_()
    dims, a = layer_inputs(wl, t)
    bufs = runner.dsa_layer(dims, **a)
    torch.cuda.synchronize()
    sel = bufs.idx.cpu().numpy()
    for b in range(wl.batch):
        for tt in range(wl.n_q):
            cand = O.visible_keys(int(wl["q_pos"][b, tt]), int(wl["kv_start"][b]), int(wl["kv_len"][b]))
            want = cand[:top_k].tolist()
            assert sel[b, tt].tolist() == want + [O.INVALID] * (top_k - len(want)), (b, tt)


# ------------------------------------------------ S8 absorption GEMMs
@pytest.mark.parametrize("n_rows,H", [(128, 2), (300, 4), (1400, 16)])
def test_absorb_gemms_match_oracle_and_cuda_core_kernel(n_rows, H):
    # ragged row counts (several 128-row tiles and a tail); at 1400 x 16 a CTA takes 2-3 items
    # and some ranges cross a head boundary (B reloaded, both accumulators in turn)
    g = torch.Generator().manual_seed(n_rows + H)
    q = (torch.randn(n_rows, H, 128, generator=g)).to(torch.bfloat16)
    o_lat = (torch.randn(n_rows, H, 512, generator=g)).to(torch.bfloat16)
    w_uk = (torch.randn(H, 128, 512, generator=g) / 512 ** 0.5).to(torch.bfloat16)
    w_uv = (torch.randn(H, 128, 512, generator=g) / 512 ** 0.5).to(torch.bfloat16)
    d = dsa.Dims(batch=1, n_q=n_rows, heads=H, dtype=dsa.BF16)
    qd, od, ukd, uvd = (x.cuda() for x in (q, o_lat, w_uk, w_uv))
    outs = {}
    for policy in (0, 1):
        prev = dsa.set_kernel_policy(policy)
        try:
            q_lat = torch.full((n_rows, H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
            out = torch.full((n_rows, H, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
            dsa.absorb_q(d, qd, 128, ukd, 512, q_lat)
            dsa.absorb_out(d, od, 512, uvd, 128, out)
            torch.cuda.synchronize()
            outs[policy] = (q_lat.double().cpu().numpy(), out.double().cpu().numpy())
        finally:
            dsa.set_kernel_policy(prev)
    ref_q = O.absorb_q(q.float().numpy(), w_uk.float().numpy())
    ref_o = O.absorb_out(o_lat.float().numpy(), w_uv.float().numpy())
    for policy, (gq, go) in outs.items():
        # fp32 accumulation of bf16 products, one bf16 rounding of the result
        np.testing.assert_allclose(gq, ref_q, atol=2e-2, rtol=1e-2, err_msg=f"absorb_q policy {policy}")
        np.testing.assert_allclose(go, ref_o, atol=2e-2, rtol=1e-2, err_msg=f"absorb_out policy {policy}")
    # the two kernel families differ only in summation order
    np.testing.assert_allclose(outs[0][0], outs[1][0], atol=1e-2, rtol=1e-2)
    np.testing.assert_allclose(outs[0][1], outs[1][1], atol=1e-2, rtol=1e-2)


# ------------------------------------------- tensor cores vs CUDA cores
@pytest.mark.parametrize("name,sizes,top_k", [("prefill", dict(T=300), 96), ("decode", dict(B=2, S=4100), 2048)])
def test_tensor_core_kernels_match_cuda_core_kernels(name, sizes, top_k):
    """Same inputs through both kernel families (dsa_set_kernel_policy)."""
    wl = workloads.make(name, **sizes)
    wl.top_k = top_k
    t = dev(wl)
    try:
        dsa.set_kernel_policy(1)
        _, _, sc_simt, idx_simt, _, out_simt, lse_simt = _run_stages(wl, t)
        dsa.set_kernel_policy(0)
        _, _, sc_tc, idx_tc, _, out_tc, lse_tc = _run_stages(wl, t)
    finally:
        dsa.set_kernel_policy(0)
    fin = torch.isfinite(sc_simt)
    assert torch.equal(fin, torch.isfinite(sc_tc))
    scale_ = sc_simt[fin].abs().max().clamp(min=1.0)
    assert (sc_simt[fin] - sc_tc[fin]).abs().max() <= 2e-5 * scale_
    # attend both families over the same selection
    dims, a = layer_inputs(wl, t)
    outs = []
    for pol in (1, 0):
        dsa.set_kernel_policy(pol)
        o = torch.empty_like(out_tc)
        l = torch.empty_like(lse_tc)
        dsa.sparse_attend(dims, a["q"], a["k"], a["k_row_stride"], a["v"], a["v_row_stride"], idx_simt,
                          wl.top_k, a["attn_scale"], o, l)
        outs.append((o, l))
    dsa.set_kernel_policy(0)
    torch.cuda.synchronize()
    assert_attend_close(_np(outs[1][0]), _np(outs[0][0]), torch.bfloat16, "tc vs simt attend", gpu_pair=True)
    assert (outs[1][1] - outs[0][1]).abs().max().item() <= 2e-3


# ------------------------------------------------- caches past 16-bit key indices
def test_long_cache_layer_stays_on_tensor_cores():
    """A 70000-key cache (past 65536, where a key index needs more than 16 bits): the fused layer
    still runs on the tensor cores (the fused selection, then attend_tc), and every row matches the
    oracle."""
    S = 70000
    wl = workloads.make("decode", B=3, S=S)
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    bufs = runner.LayerBuffers(dims, "cuda", torch.bfloat16, with_idx=True, with_lse=True)
    runner.dsa_layer(dims, **a, bufs=bufs)
    assert dsa.last_kernels() == ["index_topk", "attend_tc"]
    scores = torch.empty(3, 1, S, dtype=torch.float32, device="cuda")
    dsa.index_scores(dims, t["q_idx"], t["k_idx"], t["w"], wl.idx_scale, t["q_pos"], t["kv_start"], t["kv_len"], scores)
    torch.cuda.synchronize()
    g_idx, g_out, g_lse = bufs.idx.cpu().numpy(), _np(bufs.out), bufs.lse.cpu().numpy()
    assert int((bufs.idx > 65535).sum()) > 100           # the selection reaches past 16 bits
    K, V = kv_views(wl)
    for b in range(3):
        cand = O.visible_keys(S - 1, 0, S)
        ref = O.index_scores_row(wl["q_idx"][b, 0], wl["k_idx"][b], wl["w"][b, 0], wl.idx_scale)
        gs = scores[b, 0].cpu().numpy().astype(np.float64)
        assert np.abs(gs - ref).max() <= 2e-5 * max(1.0, np.abs(ref).max())
        assert g_idx[b, 0].tolist() == key_order(O.topk_row(cand, gs, wl.top_k).tolist())
        check_selection_in_band(g_idx[b, 0], cand, ref, wl.top_k, f"long cache row {b}")
        ro, rl = O.sparse_attend_row(wl["q"][b, 0], K[b], V[b], g_idx[b, 0], wl.attn_scale)
        assert_attend_close(g_out[b, 0], ro, torch.bfloat16, f"long cache out {b}")
        np.testing.assert_allclose(g_lse[b, 0], rl, atol=2e-3)


@pytest.mark.parametrize("H,kd", [(128, 576), (64, 512)])
def test_long_cache_attend_set_semantics(H, kd):
    """dsa_sparse_attend on the tensor cores over a 70000-row latent with index rows that mix keys
    above and below 65536, duplicates (the first-occurrence compaction), INVALID and out-of-range
    entries, against the oracle's set-semantics attention; rows 100 and T-1 run as a cluster's second
    or third row."""
    rng = np.random.default_rng(H)
    # more rows than the kernel's 74 persistent clusters, so clusters run a second and a third row
    B, T, S, W = 1, 130 if H == 64 else 150, 70000, 2048
    q = torch.tensor(rng.standard_normal((B, T, H, kd)), dtype=torch.bfloat16)
    lat = torch.tensor(rng.standard_normal((B, S, kd)) * 0.5, dtype=torch.bfloat16)
    idx = rng.integers(0, S, size=(B, T, W)).astype(np.int32)
    idx[0, 0, ::5] = O.INVALID
    idx[0, 1, 1024:] = idx[0, 1, :1024]                   # duplicates
    idx[0, 2, ::9] = S + 5                                # out of range
    idx[0, 3, :] = np.arange(65536 - 1024, 65536 + 1024)  # straddles the 16-bit boundary
    d = dsa.Dims(batch=B, n_q=T, n_kv=S, heads=H, kv_heads=1, kd=kd, vd=512, top_k=W, dtype=dsa.BF16)
    out = torch.empty(B, T, H, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, T, H, dtype=torch.float32, device="cuda")
    ld = lat.cuda()
    dsa.sparse_attend(d, q.cuda(), ld, kd, ld, kd, torch.tensor(idx).cuda(), W, 0.07, out, lse)
    assert dsa.last_kernels() == ["attend_tc"]
    torch.cuda.synchronize()
    K, V = lat.unsqueeze(2), lat[..., :512].unsqueeze(2)
    rows = range(T) if T <= 8 else list(range(6)) + [64, 100, T - 1]
    for tt in rows:
        ro, rl = O.sparse_attend_row(q[0, tt], K[0], V[0], idx[0, tt], 0.07)
        assert_attend_close(_np(out[0, tt]), ro, torch.bfloat16, f"wide attend H{H} row {tt}")
        np.testing.assert_allclose(lse[0, tt].cpu().numpy(), rl, atol=2e-3)


# ------------------------------------------------------------- kpool (small)
def _kpool_run(wl):
    t = dev(wl)
    B, T, S = wl.batch, wl.n_q, wl.n_kv
    H, L = wl.heads, wl.kd
    dims = runner.kpool_dims(B, T, S, wl.idx_heads, wl.idx_dim, wl.kpool, wl.select_k, wl.out_width, H, L)
    bufs = runner.KpoolBuffers(B, T, S, wl.idx_heads, wl.idx_dim, wl.kpool, wl.select_k, wl.out_width,
                               H, t["q_nope"].shape[-1], L, t["w_uv"].shape[1], "cuda")
    runner.kpool_layer(dims, t["q_idx"], t["k_raw"], t["gate"], t["ln_w"], t["ln_b"], wl.ln_eps, t["w"],
                       wl.idx_scale, t["q_pos"], t["kv_start"], t["kv_len"], t["q_nope"], t["latent"],
                       t["w_uk"], t["w_uv"], wl.attn_scale, bufs)
    torch.cuda.synchronize()
    return bufs


def _kpool_check(wl, bufs, rows):
    B = wl.batch
    kp = wl.kpool
    npools = bufs.n_pools.cpu().tolist()
    pooled = bufs.pooled.float().cpu().numpy()
    pool_scores = bufs.pool_scores.cpu().numpy().astype(np.float64)
    pool_idx = bufs.pool_idx.cpu().numpy()
    tok_idx = bufs.tok_idx.cpu().numpy()
    out = _np(bufs.out)
    q_lat = _np(bufs.q_lat)
    refpool = {}
    worst = (1.0, 0.0)
    for b in range(B):
        f, L = int(wl["kv_start"][b]), int(wl["kv_len"][b])
        assert npools[b] == O.n_pools_of(f, L, kp)
        ref = O.pool_states(wl["k_raw"][b], wl["gate"][b], f, L, kp, wl["ln_w"], wl["ln_b"], wl.ln_eps)
        refpool[b] = ref
        np.testing.assert_allclose(pooled[b, :npools[b]], ref, atol=3e-2, rtol=1e-2)
        assert np.all(pooled[b, npools[b]:] == 0)
    for b, tt in rows:
        f = int(wl["kv_start"][b])
        L = int(wl["kv_len"][b])
        p = int(wl["q_pos"][b, tt])
        cand = O.visible_pools(p, f, npools[b], kp)
        # index over the GPU's pooled keys (bf16 values as stored), oracle arithmetic
        gpk = bufs.pooled[b].cpu()
        ref_sc = O.index_scores_row(wl["q_idx"][b, tt], gpk[cand], wl["w"][b, tt], wl.idx_scale) \
            if cand.size else np.zeros(0)
        if cand.size:
            assert np.abs(pool_scores[b, tt, cand] - ref_sc).max() <= 2e-5 * max(1, np.abs(ref_sc).max())
        # the layer selects its pools as a set, listed in pool order (dsa_topk_set)
        assert pool_idx[b, tt].tolist() == key_order(O.topk_row(cand, pool_scores[b, tt, cand], wl.select_k).tolist())
        check_selection_in_band(pool_idx[b, tt], cand, ref_sc, wl.select_k, f"kpool pools {(b, tt)}")
        want_tok = O.expand_selection(pool_idx[b, tt], p, f, L, kp, npools[b], wl.out_width)
        assert tok_idx[b, tt].tolist() == want_tok.tolist()
        # absorbed attention over the GPU's token rows vs the literal expand_kv form
        ro, _ = O.mla_masked_attention_row(wl["q_nope"][b, tt], wl["latent"][b], wl["w_uk"], wl["w_uv"],
                                           tok_idx[b, tt], wl.attn_scale)
        c, r = assert_attend_close(out[b, tt], ro, torch.bfloat16, f"kpool out {(b, tt)}")
        worst = (min(worst[0], c), max(worst[1], r))
        np.testing.assert_allclose(q_lat[b, tt], O.absorb_q(wl["q_nope"][b, tt][None], wl["w_uk"])[0],
                                   atol=3e-2, rtol=1e-2)
    report(f"kpool T={wl.n_q}", rows=len(rows), worst_cosine=f"{worst[0]:.7f}",
           worst_maxabs_over_rms=f"{worst[1]:.4f}")


def test_kpool_small_against_oracle():
    wl = workloads.make("kpool", T=160, pads=(0, 3, 17, 70))
    wl.select_k = 8
    wl.top_k = 8
    wl.out_width = 8 * 4 + 3
    bufs = _kpool_run(wl)
    rows = [(b, t) for b in range(wl.batch) for t in range(0, wl.n_q, 7)] + [(3, 69), (3, 70), (2, 20)]
    _kpool_check(wl, bufs, rows)


# --------------------------------------------------------- full-size workloads
def _full_layer(name):
    wl = workloads.make(name)
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    bufs = runner.LayerBuffers(dims, "cuda", t["q"].dtype, with_idx=True, with_lse=True)
    runner.dsa_layer(dims, **a, bufs=bufs)
    torch.cuda.synchronize()
    return wl, t, dims, bufs


@pytest.mark.parametrize("name", ["prefill", "decode", "chunked"])
def test_full_size_layer_sampled_rows(name):
    """The workloads bench.py times, in its launch configuration: 256 sampled query rows (every
    row of decode's 64) against the oracle element by element, structure on every row."""
    wl, t, dims, bufs = _full_layer(name)
    B, T, S = wl.batch, wl.n_q, wl.n_kv
    if T == 1:
        # decode: the layer selected with the fused kernel and wrote no scores; score separately
        assert dsa.last_kernels() == ["index_topk", "attend_tc"]
        scores = torch.empty(B, T, S, dtype=torch.float32, device="cuda")
        dsa.index_scores(dims, t["q_idx"], t["k_idx"], t["w"], wl.idx_scale, t["q_pos"], t["kv_start"], t["kv_len"],
                         scores)
        torch.cuda.synchronize()
    else:
        assert dsa.last_kernels() == ["index_tc", "topk_set", "attend_tc"]
        scores = bufs.ws[: B * T * S * 4].view(torch.float32).view(B, T, S)
    g_idx = bufs.idx.cpu().numpy()
    g_out = bufs.out.cpu()
    g_lse = bufs.lse.cpu().numpy()
    K, V = kv_views(wl)
    rows = [(b, tt) for b in range(B) for tt in range(T)] if B * T <= 256 else sample_rows(wl, 256)
    diffs = 0
    worst_cos, worst_rel, worst_idx = 1.0, 0.0, 0.0
    for b, tt in rows:
        p, ks, kl = int(wl["q_pos"][b, tt]), int(wl["kv_start"][b]), int(wl["kv_len"][b])
        cand = O.visible_keys(p, ks, kl)
        ref = O.index_scores_row(wl["q_idx"][b, tt], wl["k_idx"][b][cand], wl["w"][b, tt], wl.idx_scale)
        gs = scores[b, tt].cpu().numpy().astype(np.float64)[cand]
        err = np.abs(gs - ref).max() / max(1.0, np.abs(ref).max())
        assert err <= 2e-5, (b, tt, err)
        worst_idx = max(worst_idx, err)
        assert g_idx[b, tt].tolist() == key_order(O.topk_row(cand, gs, wl.top_k).tolist())
        diffs += check_selection_in_band(g_idx[b, tt], cand, ref, wl.top_k, f"{name} {(b, tt)}") > 0
        ro, rl = O.sparse_attend_row(wl["q"][b, tt], K[b], V[b], g_idx[b, tt], wl.attn_scale)
        c, r = assert_attend_close(_np(g_out[b, tt]), ro, torch.bfloat16, f"{name} out {(b, tt)}")
        worst_cos, worst_rel = min(worst_cos, c), max(worst_rel, r)
        np.testing.assert_allclose(g_lse[b, tt], rl, atol=2e-3)
    assert diffs <= max(1, len(rows) // 4)
    report(f"full {name}", rows=len(rows), index_err_over_scale=f"{worst_idx:.2e}", rows_in_tie_band=diffs,
           worst_cosine=f"{worst_cos:.7f}", worst_maxabs_over_rms=f"{worst_rel:.4f}")
    # every row: count, visibility, ascending key order, and the same set dsa_topk ranks
    sel = bufs.idx
    qp = t["q_pos"].view(B, T, 1).long()
    valid = sel >= 0
    nvis = (qp[..., 0] - t["kv_start"].view(B, 1).long() + 1).clamp(min=0).clamp(max=S)
    assert torch.equal(valid.sum(-1), nvis.clamp(max=wl.top_k))
    assert bool((sel[valid].long() <= qp.expand_as(sel)[valid]).all())
    assert bool((sel[..., 1:][valid[..., 1:]] > sel[..., :-1][valid[..., 1:]]).all())
    ranked = torch.empty_like(sel)
    dsa.topk(dims, scores, t["q_pos"], t["kv_start"], t["kv_len"], wl.top_k, ranked)
    torch.cuda.synchronize()
    assert torch.equal(key_order(ranked), sel)


def test_ragged_batch_with_a_fully_padded_sequence():
    # three causal sequences in one batch on the tensor-core path: no padding, 37 left-padded keys with a
    # shorter cache, and one whose queries all precede its first valid key (every row selects nothing)
    T, top_k = 300, 96
    parts = [workloads.make("prefill", seed=21 + b, T=T) for b in range(3)]
    wl = parts[0]
    wl.tensors = {k: torch.cat([w.tensors[k] for w in parts], 0) for k in parts[0].tensors}
    wl.batch, wl.top_k = 3, top_k
    wl.tensors["kv_start"] = torch.tensor([0, 37, T + 5], dtype=torch.int32)
    wl.tensors["kv_len"] = torch.tensor([T, T - 50, T], dtype=torch.int32)
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    bufs = runner.LayerBuffers(dims, "cuda", torch.bfloat16, with_idx=True, with_lse=True)
    runner.dsa_layer(dims, **a, bufs=bufs)
    torch.cuda.synchronize()
    scores = bufs.ws[: 3 * T * T * 4].view(torch.float32).view(3, T, T)
    g_idx, g_out, g_lse = bufs.idx.cpu().numpy(), _np(bufs.out), bufs.lse.cpu().numpy()
    K, V = kv_views(wl)
    # the fully padded sequence: no selection, zero output, lse = -inf
    assert np.all(g_idx[2] == O.INVALID) and np.all(g_out[2] == 0) and np.all(np.isneginf(g_lse[2]))
    rows = [(0, 0), (0, top_k - 1), (0, top_k), (0, T - 1), (1, 0), (1, 36), (1, 37), (1, 38), (1, 37 + top_k),
            (1, T - 51), (1, T - 50), (1, T - 1)]
    for b, tt in rows:
        p, ks, kl = int(wl["q_pos"][b, tt]), int(wl["kv_start"][b]), int(wl["kv_len"][b])
        cand = O.visible_keys(p, ks, kl)
        if len(cand) == 0:
            assert np.all(g_idx[b, tt] == O.INVALID) and np.all(g_out[b, tt] == 0), (b, tt)
            assert np.all(np.isneginf(g_lse[b, tt])), (b, tt)
            continue
        gs = scores[b, tt].cpu().numpy().astype(np.float64)[cand]
        ref = O.index_scores_row(wl["q_idx"][b, tt], wl["k_idx"][b][cand], wl["w"][b, tt], wl.idx_scale)
        assert np.abs(gs - ref).max() <= 2e-5 * max(1.0, np.abs(ref).max()), (b, tt)
        assert g_idx[b, tt].tolist() == key_order(O.topk_row(cand, gs, top_k).tolist()), (b, tt)
        check_selection_in_band(g_idx[b, tt], cand, ref, top_k, f"ragged {(b, tt)}")
        ro, rl = O.sparse_attend_row(wl["q"][b, tt], K[b], V[b], g_idx[b, tt], wl.attn_scale)
        assert_attend_close(g_out[b, tt], ro, torch.bfloat16, f"ragged out {(b, tt)}")
        np.testing.assert_allclose(g_lse[b, tt], rl, atol=2e-3)


def test_full_size_kpool_sampled_rows():
    wl = workloads.make("kpool")
    bufs = _kpool_run(wl)
    rows = sample_rows(wl, 256, extra=[(3, 1028), (3, 1029), (1, 20)])
    _kpool_check(wl, bufs, rows)


# ----------------------------------------------------------- run properties
def test_rerun_is_bit_identical():
    wl = workloads.make("prefill", T=1024)
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    b1 = runner.dsa_layer(dims, **a)
    o1, i1 = b1.out.clone(), b1.idx.clone()
    b2 = runner.dsa_layer(dims, **a)
    torch.cuda.synchronize()
    assert torch.equal(i1, b2.idx)
    assert torch.equal(o1, b2.out)


def test_multi_sequence_batch_equals_sequences_alone():
    wl = workloads.make("decode", B=4, S=3000)
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    whole = runner.dsa_layer(dims, **a)
    torch.cuda.synchronize()
    for b in range(wl.batch):
        one = {k: (v[b:b + 1] if isinstance(v, torch.Tensor) else v) for k, v in a.items()}
        d1 = dsa.Dims(**{**dims.as_dict(), "batch": 1})
        alone = runner.dsa_layer(d1, **one)
        torch.cuda.synchronize()
        assert torch.equal(alone.idx[0], whole.idx[b])
        assert torch.equal(alone.out[0], whole.out[b])


def test_index_share_attends_over_a_foreign_selection():
    """IndexShare (ik_llama.cpp PR #2063): idx_in is another layer's selection.  Here it is the
    oracle's top-k over a different seed's indexer inputs, with INVALID padding, repeated keys,
    out-of-range entries and an empty row planted in it; the fused layer must skip S2/S3 (its own
    indexer inputs are never read, idx_out is never written) and attend over that selection as a
    set, equal to the oracle's attention row by row."""
    T, top_k = 300, 96
    wl = workloads.make("prefill", T=T)
    other = workloads.make("prefill", seed=77, T=T)
    wl.top_k = top_k
    ref_scores = O.index_scores(other["q_idx"], other["k_idx"], other["w"], other.idx_scale, other["q_pos"],
                                other["kv_start"], other["kv_len"])
    sel = O.topk(ref_scores, top_k, other["q_pos"], other["kv_start"], other["kv_len"]).astype(np.int32)
    sel[0, 120:130, 80:] = O.INVALID                          # padding inside a full row
    sel[0, 130:140, 48:] = sel[0, 130:140, :48]               # every key twice
    sel[0, 140:150, ::7] = T + 13                             # out of range
    sel[0, 150] = O.INVALID                                   # empty row
    sel[0, 151, :] = sel[0, 151, 0]                           # one key, repeated
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    a["q_idx"] = torch.full_like(a["q_idx"], float("nan"))   # must not be read
    idx_in = torch.tensor(sel).cuda()
    bufs = runner.LayerBuffers(dims, "cuda", torch.bfloat16, with_idx=True, with_lse=True)
    bufs.idx.fill_(12345)
    runner.dsa_layer(dims, **a, bufs=bufs, idx_in=idx_in)
    assert dsa.last_kernels() == ["attend_tc"]
    torch.cuda.synchronize()
    assert bool((bufs.idx == 12345).all())
    K, V = kv_views(wl)
    g_out, g_lse = _np(bufs.out), bufs.lse.cpu().numpy()
    worst = (1.0, 0.0)
    for tt in range(T):
        ro, rl = O.sparse_attend_row(wl["q"][0, tt], K[0], V[0], sel[0, tt], wl.attn_scale)
        if tt == 150:
            assert np.all(g_out[0, tt] == 0) and np.all(np.isneginf(g_lse[0, tt]))
            continue
        c, r = assert_attend_close(g_out[0, tt], ro, torch.bfloat16, f"foreign selection row {tt}")
        worst = (min(worst[0], c), max(worst[1], r))
        np.testing.assert_allclose(g_lse[0, tt], rl, atol=2e-3)
    report("index share, foreign selection", rows=T, worst_cosine=f"{worst[0]:.7f}",
           worst_maxabs_over_rms=f"{worst[1]:.4f}")
    # the same rows through dsa_sparse_attend: identical bits
    again = torch.empty_like(bufs.out)
    dsa.sparse_attend(dims, a["q"], a["k"], a["k_row_stride"], a["v"], a["v_row_stride"], idx_in, top_k,
                      a["attn_scale"], again)
    torch.cuda.synchronize()
    assert torch.equal(again, bufs.out)


def test_index_share_stack_follows_the_layer_schedule():
    """A 7-layer stack under IndexShare: layers 0, 1, 2 and 6 run their own indexer and top-k (il <= 1
    or il % 4 == 2), layers 3-5 reuse layer 2's selection.  Each layer has its own inputs; every
    layer's output equals the oracle's attention over the selection that layer used, and each
    computing layer's selection is its own indexer's (within the tie band of the oracle scores)."""
    T, top_k = 200, 64
    layers, wls = [], []
    for il in range(7):
        wl = workloads.make("prefill", seed=100 + il, T=T)
        wl.top_k = top_k
        t = dev(wl)
        dims, a = layer_inputs(wl, t)
        layers.append((dims, a))
        wls.append(wl)
    outs = runner.index_share_stack(layers)
    torch.cuda.synchronize()
    assert [runner.computes_own_selection(il) for il in range(7)] == [True, True, True, False, False, False, True]
    assert outs[3].idx is outs[2].idx and outs[5].idx is outs[2].idx and outs[6].idx is not outs[2].idx
    for il, (wl, b) in enumerate(zip(wls, outs)):
        g_idx, g_out = b.idx.cpu().numpy(), _np(b.out)
        K, V = kv_views(wl)
        for tt in (0, 63, 64, 117, T - 1):
            if runner.computes_own_selection(il):
                cand = O.visible_keys(tt, 0, T)
                ref = O.index_scores_row(wl["q_idx"][0, tt], wl["k_idx"][0][cand], wl["w"][0, tt], wl.idx_scale)
                check_selection_in_band(g_idx[0, tt], cand, ref, top_k, f"layer {il} row {tt}")
            ro, _ = O.sparse_attend_row(wl["q"][0, tt], K[0], V[0], g_idx[0, tt], wl.attn_scale)
            assert_attend_close(g_out[0, tt], ro, torch.bfloat16, f"layer {il} row {tt}")


def test_bounded_wait_expires_and_reports_timeout():
    assert dsa.get_device_status() == 0
    dsa.selftest_wait_timeout(2_000_000)      # 2 ms
    assert dsa.get_device_status() == 5       # DSA_ERR_TIMEOUT, context still usable
    assert dsa.get_device_status() == 0       # cleared
    x = torch.ones(4, device="cuda") * 2
    assert x.sum().item() == 8


# ------------------------------------------- fused indexer -> top-k (no score matrix)
@pytest.mark.parametrize("name,sizes,top_k", [("decode", dict(B=5, S=32768), 2048), ("decode", dict(B=3, S=5000), 2048),
                                              ("decode", dict(B=2, S=70000), 2048), ("prefill", dict(T=300), 96),
                                              ("chunked", dict(T=40, S=4500), 512)])
def test_fused_index_topk_equals_scores_then_topk_set(name, sizes, top_k):
    """dsa_index_topk (one cluster per query row: scores in shared memory, radix select across the
    cluster) selects exactly what dsa_index_scores + dsa_topk_set select, listed the same way, and
    writes nothing but the index rows.  Cases: decode rows of 32768 keys (two CTAs per row), short
    caches (one CTA), 70000 keys (eight CTAs), causal prefill rows with fewer visible keys than k,
    and a chunked offset with hot spots."""
    wl = workloads.make(name, **sizes)
    wl.top_k = top_k
    t = dev(wl)
    dims, a = layer_inputs(wl, t)
    B, T, S = wl.batch, wl.n_q, wl.n_kv
    fused = torch.full((B, T, top_k), 12345, dtype=torch.int32, device="cuda")
    dsa.index_topk(dims, a["q_idx"], a["k_idx"], a["w"], a["idx_scale"], a["q_pos"], a["kv_start"], a["kv_len"],
                   top_k, fused)
    assert dsa.last_kernels() == ["index_topk"]
    scores = torch.empty(B, T, S, dtype=torch.float32, device="cuda")
    dsa.index_scores(dims, a["q_idx"], a["k_idx"], a["w"], a["idx_scale"], a["q_pos"], a["kv_start"], a["kv_len"],
                     scores)
    ref = torch.empty_like(fused)
    dsa.topk_set(dims, scores, a["q_pos"], a["kv_start"], a["kv_len"], top_k, ref)
    torch.cuda.synchronize()
    if T == 1:
        # one query per row: the same tcgen05 tile shape as the standalone indexer, identical scores
        assert torch.equal(fused, ref)
    else:
        # several queries per tile in the standalone indexer: compare each row against the oracle
        g = fused.cpu().numpy()
        for b, tt in sample_rows(wl, 24):
            cand = O.visible_keys(int(wl["q_pos"][b, tt]), int(wl["kv_start"][b]), int(wl["kv_len"][b]))
            r = O.index_scores_row(wl["q_idx"][b, tt], wl["k_idx"][b][cand], wl["w"][b, tt], wl.idx_scale)
            check_selection_in_band(g[b, tt], cand, r, top_k, f"fused {name} {(b, tt)}")
            assert g[b, tt].tolist() == key_order(g[b, tt].tolist())
        n_same = int((fused == ref).all(-1).sum())
        report(f"fused index_topk {name}", rows=B * T, rows_equal_to_unfused=n_same)


def test_fused_index_topk_is_exact_on_integer_scores():
    """Integer indexer inputs (exact scores, many ties at the k-th score) at decode and prefill shapes:
    the fused selection equals the oracle's top-k set bit for bit."""
    for name, sizes, top_k in (("decode", dict(B=4, S=20000), 2048), ("prefill", dict(T=400), 128)):
        wl = workloads.make(name, exact_index=True, **sizes)
        t = dev(wl)
        dims, a = layer_inputs(wl, t)
        got = torch.empty(wl.batch, wl.n_q, top_k, dtype=torch.int32, device="cuda")
        dsa.index_topk(dims, a["q_idx"], a["k_idx"], a["w"], a["idx_scale"], a["q_pos"], a["kv_start"],
                       a["kv_len"], top_k, got)
        torch.cuda.synchronize()
        ref = O.index_scores(wl["q_idx"], wl["k_idx"], wl["w"], wl.idx_scale, wl["q_pos"], wl["kv_start"],
                             wl["kv_len"])
        want = O.topk(ref, top_k, wl["q_pos"], wl["kv_start"], wl["kv_len"])
        assert torch.equal(got.cpu(), key_order(torch.tensor(want, dtype=torch.int32))), name
