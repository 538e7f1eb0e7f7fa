"""Helpers shared by the GPU parity tests: device copies of workloads, row
sampling, and the comparison rules (exact, tie-band, float tolerance)."""
from __future__ import annotations

import math
import random

import numpy as np
import torch

from oracle import dsa_oracle as O
import sparse_attention_sum_b200 as dsa
from sparse_attention_sum_b200 import runner

# Float tolerances (attention outputs): max-abs 2e-2 (bf16) / 1e-4 (fp32) and
# per-row cosine >= 0.9999.  Selection: bit-exact where scores are exact; else
# every disagreement within 1e-5 * max(|tau|, max|I|) of the k-th score tau.
ATOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}
COS_MIN = 0.9999
TIE_BAND = 1e-5
# Per row, max |diff| / RMS(reference).  bf16: the output is rounded to bf16 once (at most 2^-8
# of each element, and a row's largest element is about 5 RMS over 128 x 512 near-Gaussian
# outputs: 0.02 RMS) and each probability once (2^-8 of each weight; random over the selected
# keys, larger where a few keys dominate, as with the chunked workload's N(0,1) latent).  The
# worst rows measured on the full-size workloads sit at 0.015 (decode) to 0.063 (chunked); the
# bound is 0.1.  Two GPU results compared with each other carry both roundings twice.
REL_MAX = {torch.bfloat16: 1e-1, torch.float32: 1e-3}
REL_MAX_GPU_PAIR = {torch.bfloat16: 2e-1, torch.float32: 2e-3}


def dev(wl, device="cuda"):
    return {k: v.to(device) for k, v in wl.tensors.items()}


def layer_inputs(wl, t):
    """(dims, args) for runner.dsa_layer from a token-mode workload on device."""
    if "latent" in t:
        k = t["latent"]
        v = t["latent"]
        ks = vs = wl.kd
        kk = k
    else:
        kk = t["k"]
        v = t["v"]
        ks = wl.kv_heads * wl.kd
        vs = wl.kv_heads * wl.vd
    dims = runner.layer_dims(t["q_idx"], t["k_idx"], t["q"], kk if kk.dim() == 4 else kk, wl.vd, wl.top_k)
    dims.kv_heads = wl.kv_heads
    return dims, dict(q_idx=t["q_idx"], k_idx=t["k_idx"], w=t["w"], idx_scale=wl.idx_scale,
                      q_pos=t["q_pos"], kv_start=t["kv_start"], kv_len=t["kv_len"], q=t["q"], k=kk,
                      v=v, attn_scale=wl.attn_scale, k_row_stride=ks, v_row_stride=vs)


def kv_views(wl):
    """Oracle-side K/V caches [B,S,Hk,kd] / [B,S,Hk,vd] (views, still bf16/fp32)."""
    if "latent" in wl.tensors:
        lat = wl["latent"]
        return lat.unsqueeze(2), lat[..., :wl.vd].unsqueeze(2)
    return wl["k"], wl["v"]


def sample_rows(wl, n=12, seed=0, extra=()):
    """First, last, the top-k boundary row and evenly spread rows (b, t)."""
    B, T = wl.batch, wl.n_q
    rows = {(0, 0), (B - 1, T - 1)}
    qp = wl["q_pos"]
    ks = wl["kv_start"]
    for b in range(B):
        # first row whose visible count exceeds top_k
        for t in range(T):
            if int(qp[b, t]) - int(ks[b]) + 1 > wl.top_k:
                rows.add((b, t))
                break
    rnd = random.Random(seed)
    n = min(n, B * T)                      # a workload with fewer rows gives all of them
    while len(rows) < n:
        rows.add((rnd.randrange(B), rnd.randrange(T)))
    rows |= set(extra)
    return sorted(rows)


def cosine(a: np.ndarray, b: np.ndarray) -> float:
    na, nb = np.linalg.norm(a), np.linalg.norm(b)
    if na == 0 and nb == 0:
        return 1.0
    return float(np.dot(a.ravel(), b.ravel()) / (na * nb))


def assert_attend_close(gpu_out, ref_out, dtype, what="", gpu_pair=False):
    """gpu_out, ref_out: [..., H, vd] for one or more rows.

    Checks max |diff| <= ATOL, and per query row cosine >= COS_MIN and
    max |diff| / RMS(ref) <= REL_MAX (REL_MAX_GPU_PAIR when ``gpu_pair``: both sides are GPU
    results).  Returns the worst (smallest) cosine and the worst relative error over the rows,
    for reporting."""
    rel_max = (REL_MAX_GPU_PAIR if gpu_pair else REL_MAX)[dtype]
    g = np.asarray(gpu_out, dtype=np.float64)
    r = np.asarray(ref_out, dtype=np.float64)
    err = np.abs(g - r).max() if g.size else 0.0
    assert err <= ATOL[dtype], f"{what}: max |diff| {err} > {ATOL[dtype]}"
    gr = g.reshape(-1, g.shape[-2] * g.shape[-1]) if g.ndim >= 2 else g.reshape(1, -1)
    rr = r.reshape(gr.shape)
    worst_cos, worst_rel = 1.0, 0.0
    for i in range(gr.shape[0]):
        rms = float(np.sqrt(np.mean(rr[i] ** 2)))
        if rms > 0:
            c = cosine(gr[i], rr[i])
            rel = float(np.abs(gr[i] - rr[i]).max()) / rms
            assert c >= COS_MIN, f"{what}: row {i} cosine {c}"
            assert rel <= rel_max, f"{what}: row {i} max|diff|/RMS {rel} > {rel_max}"
            worst_cos, worst_rel = min(worst_cos, c), max(worst_rel, rel)
    return worst_cos, worst_rel


def report(name, **vals):
    """One line of figures for the test log (run pytest with -s to see them)."""
    print(f"[parity] {name}: " + ", ".join(f"{k}={v}" for k, v in vals.items()))


def key_order(sel):
    """Selection rows [..., k] listed in ascending key order, DSA_INVALID after the keys
    (how dsa_layer_forward lists the set that dsa_topk ranks)."""
    if isinstance(sel, torch.Tensor):
        big = torch.iinfo(torch.int32).max
        s = torch.sort(sel.masked_fill(sel < 0, big), dim=-1).values
        return s.masked_fill(s == big, O.INVALID)
    keys = sorted(int(x) for x in sel if int(x) != O.INVALID)
    return keys + [O.INVALID] * (len(sel) - len(keys))


def check_selection_in_band(gpu_sel, cand, ref_scores, k, what=""):
    """GPU selection vs the oracle's scores: equal, or every difference inside the tie band.

    Returns the number of differing keys (0 when the rows are identical).
    """
    ref_sel = O.topk_row(cand, ref_scores, k)
    g = [int(x) for x in gpu_sel]
    r = [int(x) for x in ref_sel]
    if g == r:
        return 0
    n_valid = min(k, len(cand))
    assert sum(1 for x in g if x != O.INVALID) == n_valid, f"{what}: selected count"
    assert all(x == O.INVALID for x in g[n_valid:]), f"{what}: INVALID tail"
    gs, rs = set(g[:n_valid]), set(r[:n_valid])
    score_of = dict(zip(cand.tolist(), ref_scores.tolist()))
    tau = score_of[r[n_valid - 1]]
    scale_ = max(abs(tau), max(abs(x) for x in ref_scores.tolist()))
    band = TIE_BAND * scale_
    for key in gs ^ rs:
        assert key in score_of, f"{what}: selected key {key} not visible"
        assert abs(score_of[key] - tau) <= band, \
            f"{what}: key {key} score {score_of[key]} outside tie band {band} of tau {tau}"
    # the ranked order agrees up to swaps inside the band
    return len(gs ^ rs)
