"""Pins for the CPU oracle (no GPU).

Each test fixes part of the oracle to something other than the oracle itself:
hand-worked values from the pages (``tests/golden``), closed forms,
invariants the pages state, special cases that reduce to a library routine,
exact rational arithmetic, or brute force on tiny inputs.  The last test
plants mistakes in a copy of the oracle and checks that the pins catch them.
"""
import json
import math
import os
import random
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import dsa_oracle as O
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- P1 hand case
def test_hand_index_scores_and_topk():
    g = _golden("hand_index_topk.json")
    q = np.array(g["q"])
    keys = np.array(g["keys"])
    w = np.array(g["w"])
    sc = O.index_scores_row(q, keys, w, g["idx_scale"])
    assert sc.tolist() == g["scores_pos3"]
    for case in g["cases"]:
        cand = O.visible_keys(case["q_pos"], 0, len(keys))
        s = O.index_scores_row(q, keys[cand], w, g["idx_scale"])
        got = O.topk_row(cand, s, case["k"])
        assert got.tolist() == case["expect"], case


def test_visibility_rules():
    # causal inclusive, padding, and kv_len bound
    assert O.visible_keys(5, 0, 10).tolist() == [0, 1, 2, 3, 4, 5]
    assert O.visible_keys(5, 3, 10).tolist() == [3, 4, 5]
    assert O.visible_keys(2, 3, 10).tolist() == []          # padded query row
    assert O.visible_keys(12, 0, 8).tolist() == list(range(8))
    # pools: only complete, causally visible pools
    assert O.visible_pools(6, 0, 10, 4).tolist() == [0]
    assert O.visible_pools(7, 0, 10, 4).tolist() == [0, 1]
    assert O.visible_pools(7, 0, 1, 4).tolist() == [0]
    assert O.visible_pools(2, 3, 10, 4).tolist() == []


# ------------------------------------------------------- P2 dense reduction
@pytest.mark.parametrize("Hk", [1, 4])
def test_topk_covering_all_keys_equals_dense_attention(Hk):
    """top_k >= visible keys turns the sparse layer into dense causal attention
    (ik_llama.cpp #2045: PPL byte-identical to dense when top_k >= n_tokens)."""
    rng = np.random.default_rng(7)
    B, T, HI, DI, H, kd, vd = 2, 13, 3, 8, 4, 10, 6
    q_idx = rng.standard_normal((B, T, HI, DI))
    k_idx = rng.standard_normal((B, T, DI))
    w = rng.standard_normal((B, T, HI))
    q = rng.standard_normal((B, T, H, kd))
    k = rng.standard_normal((B, T, Hk, kd))
    v = rng.standard_normal((B, T, Hk, vd))
    q_pos = np.tile(np.arange(T), (B, 1))
    kv_start = np.array([0, 4])
    kv_len = np.array([T, T - 2])
    wl = dict(q_idx=q_idx, k_idx=k_idx, w=w, q_pos=q_pos, kv_start=kv_start, kv_len=kv_len)
    dense = O.dense_causal_attend(q, k, v, 0.3, q_pos, kv_start, kv_len)
    for b in range(B):
        for t in range(T):
            sel, out, lse, _ = O.layer_row(b, t, wl, T, 0.25, 0.3, q, k, v)
            np.testing.assert_allclose(out, dense[b, t], rtol=0, atol=1e-12)


# --------------------------------------------------------- P3 hand attend
def test_hand_attend_sets():
    g = _golden("hand_attend.json")
    q = np.array([g["q"]])                   # one head
    K = np.array(g["keys"])[:, None, :]
    V = np.array(g["values"])[:, None, :]
    lse_map = {"0.5+ln2": 0.5 + math.log(2.0), "0.5": 0.5, "-inf": -math.inf}
    for case in g["cases"]:
        out, lse = O.sparse_attend_row(q, K, V, np.array(case["idx"]), g["scale"])
        assert out[0].tolist() == pytest.approx(case["out"], abs=1e-15)
        want = lse_map[case["lse"]]
        if math.isinf(want):
            assert math.isinf(lse[0]) and lse[0] < 0
        else:
            assert lse[0] == pytest.approx(want, abs=1e-15)


def test_softmax_two_key_closed_form():
    # weights e^a / (e^a + e^b) for logits a, b
    q = np.array([1.0, 2.0])
    K = np.array([[0.3, -0.1], [1.0, 0.25]])
    V = np.array([[1.0, 0.0, 5.0], [0.0, 1.0, -5.0]])
    a, b = 0.7 * (0.3 - 0.2), 0.7 * (1.0 + 0.5)
    pa = math.exp(a) / (math.exp(a) + math.exp(b))
    out, lse = O.attend_row(q, K, V, 0.7)
    np.testing.assert_allclose(out, [pa, 1 - pa, 5 * pa - 5 * (1 - pa)], atol=1e-15)
    assert lse == pytest.approx(math.log(math.exp(a) + math.exp(b)), abs=1e-14)


def test_dense_selection_matches_torch_sdpa():
    """With every visible key selected, the sparse attend is torch's masked SDPA."""
    rng = np.random.default_rng(3)
    T, H, kd, vd = 9, 3, 7, 5
    q = rng.standard_normal((1, T, H, kd))
    k = rng.standard_normal((1, T, H, kd))
    v = rng.standard_normal((1, T, H, vd))
    idx = np.array([[list(range(t + 1)) + [-1] * (T - t - 1) for t in range(T)]])
    out, _ = O.sparse_attend(q, k, v, idx, 0.45)
    tq = torch.tensor(q[0]).permute(1, 0, 2)
    tk = torch.tensor(k[0]).permute(1, 0, 2)
    tv = torch.tensor(v[0]).permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=0.45)
    np.testing.assert_allclose(out[0], ref.permute(1, 0, 2).numpy(), atol=1e-12)


# ------------------------------------------------------- P4 WHT invariance
def test_walsh_hadamard_rotation_leaves_scores_unchanged():
    """(Hq).(Hk) = D q.k for the unnormalised Sylvester matrix, so scale/D gives
    bit-identical f64 scores (ik_llama.cpp #2045: the orthonormal rotation
    leaves q.k unchanged)."""
    rng = np.random.default_rng(11)
    D, HI, n = 32, 4, 40
    Hm = scipy.linalg.hadamard(D).astype(np.float64)
    q = rng.integers(-4, 5, (HI, D)).astype(np.float64)
    k = rng.integers(-4, 5, (n, D)).astype(np.float64)
    w = rng.choice([0.5, 1.0, 2.0, 4.0], HI)
    base = O.index_scores_row(q, k, w, 1.0 / 8.0)
    rot = O.index_scores_row(q @ Hm.T, k @ Hm.T, w, 1.0 / 8.0 / D)
    assert np.array_equal(base, rot)
    assert np.any(base > 0)


# ------------------------------------------------------ P5 brute-force top-k
def _brute_topk(cand, scores, k):
    """Repeatedly take the best remaining candidate: highest score, then smallest index."""
    remaining = list(zip(cand.tolist(), scores.tolist()))
    out = []
    while remaining and len(out) < k:
        best = None
        for i, s in remaining:
            if best is None or s > best[1] or (s == best[1] and i < best[0]):
                best = (i, s)
        out.append(best[0])
        remaining.remove(best)
    return out + [O.INVALID] * (k - len(out))


def test_topk_matches_brute_force_with_ties():
    rnd = random.Random(5)
    for trial in range(300):
        n = rnd.randint(0, 40)
        k = rnd.randint(1, 45)
        cand = np.array(sorted(rnd.sample(range(100), n)), dtype=np.int64)
        scores = np.array([rnd.choice([-1.0, -0.0, 0.0, 0.5, 1.0, 2.0]) for _ in range(n)])
        got = O.topk_row(cand, scores, k).tolist()
        assert got == _brute_topk(cand, scores + 0.0, k), (cand, scores, k)


# -------------------------------------------------- P6 exact integer scores
def test_tiny_workload_scores_are_exact_rationals():
    wl = workloads.make("tiny")
    q, k, w = wl["q_idx"][0], wl["k_idx"][0], wl["w"][0]
    for t in (0, 17, 40, 63):
        cand = O.visible_keys(t, 0, 64)
        got = O.index_scores_row(q[t], k[cand], w[t], wl.idx_scale)
        for j, s in enumerate(cand.tolist()):
            exact = Fraction(0)
            for h in range(wl.idx_heads):
                dot = sum(int(q[t, h, d]) * int(k[s, d]) for d in range(wl.idx_dim))
                exact += Fraction(w[t, h].item()) * max(Fraction(0), Fraction(dot, 8))
            assert Fraction(got[j]) == exact
            assert (exact * 16).denominator == 1          # multiples of 1/16
            assert abs(exact) <= 1024


# -------------------------------------------------------- P7 pooling cases
def test_pooling_starts_at_first_valid_token_and_drops_partial_pool():
    g = _golden("hand_kpool.json")
    kp = g["kpool"]
    rng = np.random.default_rng(2)
    for case in g["pooling"]:
        n = case["kv_len"]
        k = rng.standard_normal((n, 6))
        gate = np.zeros((n, 6))                     # constant gate: slot mean
        assert O.n_pools_of(case["kv_start"], n, kp) == case["n_pools"]
        assert O.kept_pools(case["kv_start"], n, kp).tolist() == list(range(case["n_pools"]))
        pooled = O.pool_states(k, gate, case["kv_start"], n, kp, None, None, 1e-6)
        toks = case["pool0_tokens"]
        want = O.layer_norm(k[toks], None, None, 1e-6).mean(axis=0)
        np.testing.assert_allclose(pooled[0], want, atol=1e-14)


def test_pool_gate_softmax_is_per_channel_over_slots():
    rng = np.random.default_rng(4)
    k = rng.standard_normal((8, 3))
    gate = np.zeros((8, 3))
    gate[5, 0] = 60.0       # slot 1 of pool 1 dominates channel 0 only
    gate[6, 2] = 60.0       # slot 2 of pool 1 dominates channel 2 only
    pooled = O.pool_states(k, gate, 0, 8, 4, None, None, 1e-6)
    kn = O.layer_norm(k, None, None, 1e-6)
    assert pooled[1, 0] == pytest.approx(kn[5, 0], abs=1e-20 + 1e-12)
    assert pooled[1, 2] == pytest.approx(kn[6, 2], abs=1e-12)
    assert pooled[1, 1] == pytest.approx(kn[4:8, 1].mean(), abs=1e-14)


def test_pool_topk_matches_brute_force_over_fully_visible_pools():
    """topk_pools_row against brute force on tiny inputs: every pool is scored from the pooled keys one
    (query head, pool) dot at a time, a pool is a candidate only when all its kpool tokens lie between
    the first valid token and the query (the pages' 'valid only if all kpool slots are valid'), and the
    candidates are ranked by a full sort on (score descending, pool id ascending).  Integer operands
    give many exact ties."""
    rng = np.random.default_rng(11)
    kp, n_pools, H, D = 4, 9, 2, 3
    pooled = rng.integers(-2, 3, size=(n_pools, D)).astype(float)
    q = rng.integers(-2, 3, size=(H, D)).astype(float)
    w = np.array([1.0, 0.5])
    for f in (0, 3):
        for q_pos in range(f - 1, f + n_pools * kp + 2):
            for sel_k in (1, 3, 12):
                got, _ = O.topk_pools_row(q, pooled, w, 0.5, q_pos, f, n_pools, kp, sel_k)
                cands = []
                for pid in range(n_pools):
                    last_token = f + pid * kp + kp - 1
                    if q_pos >= f and last_token <= q_pos:
                        score = 0.0
                        for h in range(H):
                            dot = sum(q[h, d] * pooled[pid, d] for d in range(D))
                            score += w[h] * max(0.0, 0.5 * dot)
                        cands.append((-score, pid))
                want = [pid for _, pid in sorted(cands)[:sel_k]]
                want += [O.INVALID] * (sel_k - len(want))
                assert got.tolist() == want, (f, q_pos, sel_k)


# -------------------------------------------------------- P8 expand cases
def test_expand_selection_examples():
    g = _golden("hand_kpool.json")
    kp = g["kpool"]
    for case in g["expand"]:
        npools = O.n_pools_of(case["kv_start"], case["kv_len"], kp)
        got = O.expand_selection(case["pools"], case["q_pos"], case["kv_start"], case["kv_len"],
                                 kp, npools, case["out_width"])
        assert got.tolist() == case["expect"], case["worked"]


def test_expand_selection_tail_length_and_validity():
    kp, f, L, selk = 4, 3, 40, 5
    width = selk * kp + kp - 1
    npools = O.n_pools_of(f, L, kp)
    for t in range(0, L):
        vis = O.visible_pools(t, f, npools, kp)
        pools = list(vis[::-1][:selk]) + [O.INVALID] * max(0, selk - len(vis))
        out = O.expand_selection(pools, t, f, L, kp, npools, width)
        assert out.shape == (width,)
        toks = out[out != O.INVALID]
        if t < f:
            assert toks.size == 0
            continue
        r = t - f
        tail = [s for s in toks.tolist() if s >= f + len(vis) * kp]
        assert len(tail) == (min(t, L - 1) - f + 1) - len(vis) * kp
        if (r + 1) // kp <= npools:
            assert len(tail) == (r + 1) % kp
        assert len(set(toks.tolist())) == toks.size                 # no duplicates
        assert all(f <= s <= t for s in toks.tolist())              # all visible
        assert np.all(out[toks.size:] == O.INVALID)                 # INVALID only at the end


# ------------------------------------------------ P9 absorption identity
def test_absorbed_mla_equals_literal_expand_kv():
    rng = np.random.default_rng(9)
    H, d, L, n = 3, 5, 12, 17
    q = rng.standard_normal((H, d))
    lat = rng.standard_normal((n, L))
    uk = rng.standard_normal((H, d, L)) / math.sqrt(L)
    uv = rng.standard_normal((H, d + 1, L)) / math.sqrt(L)
    row = np.array([3, 3, 16, -1, 0, 9, 40, 5])
    lit, lse1 = O.mla_masked_attention_row(q, lat, uk, uv, row, 0.4)
    ab, lse2 = O.mla_absorbed_row(q, lat, uk, uv, row, 0.4)
    np.testing.assert_allclose(lit, ab, atol=1e-10)
    np.testing.assert_allclose(lse1, lse2, atol=1e-10)
    # the batched absorb helpers agree with the per-head routine
    ql = O.absorb_q(q[None], uk)[0]
    np.testing.assert_allclose(ql[1], uk[1].T @ q[1], atol=1e-13)
    ol = O.absorb_out(np.ones((1, H, L)), uv)[0]
    np.testing.assert_allclose(ol[2], uv[2].sum(axis=1), atol=1e-13)


# ------------------------------------------------------ P10 invariances
def test_index_row_permutation_invariance():
    rng = np.random.default_rng(1)
    H, kd, vd, n = 4, 9, 7, 30
    q = rng.standard_normal((H, kd))
    K = rng.standard_normal((n, 1, kd))
    V = rng.standard_normal((n, 1, vd))
    row = rng.choice(n, 20, replace=False)
    a, la = O.sparse_attend_row(q, K, V, row, 0.5)
    b, lb = O.sparse_attend_row(q, K, V, rng.permutation(row), 0.5)
    np.testing.assert_allclose(a, b, atol=1e-12)
    np.testing.assert_allclose(la, lb, atol=1e-12)


def test_multi_sequence_batch_equals_sequences_alone():
    """ik_llama.cpp #2063 UPDATE 5: n_seq=4 equals n_seq=1 chunk for chunk."""
    rng = np.random.default_rng(8)
    B, T, HI, DI, H, kd, vd = 3, 11, 2, 6, 2, 5, 4
    ts = dict(q_idx=rng.standard_normal((B, T, HI, DI)), k_idx=rng.standard_normal((B, T, DI)),
              w=rng.standard_normal((B, T, HI)), q_pos=np.tile(np.arange(T), (B, 1)),
              kv_start=np.array([0, 2, 5]), kv_len=np.array([T, T, 9]))
    q = rng.standard_normal((B, T, H, kd))
    k = rng.standard_normal((B, T, 1, kd))
    v = rng.standard_normal((B, T, 1, vd))
    for b in range(B):
        alone = {key: (val[b:b + 1]) for key, val in ts.items()}
        for t in range(T):
            s1, o1, _, _ = O.layer_row(b, t, ts, 4, 0.3, 0.6, q, k, v)
            s2, o2, _, _ = O.layer_row(0, t, alone, 4, 0.3, 0.6, q[b:b + 1], k[b:b + 1], v[b:b + 1])
            assert s1.tolist() == s2.tolist()
            np.testing.assert_array_equal(o1, o2)


# ---------------------------------------------------------- P11 LayerNorm
def test_layer_norm_matches_torch_and_moments():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((5, 128)) * 3 + 1
    w = 1 + 0.1 * rng.standard_normal(128)
    b = 0.1 * rng.standard_normal(128)
    got = O.layer_norm(x, w, b, 1e-6)
    ref = torch.nn.functional.layer_norm(torch.tensor(x), (128,), torch.tensor(w), torch.tensor(b), 1e-6)
    np.testing.assert_allclose(got, ref.numpy(), atol=1e-12)
    plain = O.layer_norm(x, None, None, 1e-6)
    np.testing.assert_allclose(plain.mean(axis=1), 0, atol=1e-13)
    np.testing.assert_allclose(plain.var(axis=1), 1, atol=1e-5)
    with pytest.raises(ValueError):
        O.layer_norm(x, w, b, 0.0)


# ------------------------------------- P13 indexer query/key preparation
def test_rope_neox_pairs_halves_with_closed_form_angles():
    """NEOX RoPE pairs value i with value i + n_rope/2 and turns pair i by
    pos * theta^(-2i/n_rope).  n_rope = 4, theta = 10000, pos = 3: a unit vector
    on value 0 turns by 3 rad into values 0 and 2, one on value 1 by 3/100 rad
    into values 1 and 3, and value 4 (past n_rope) stays put."""
    e = np.eye(5)
    y = O.rope_neox(e, 3, 4, 10000.0)
    np.testing.assert_allclose(y[0], [math.cos(3), 0, math.sin(3), 0, 0], atol=1e-15)
    np.testing.assert_allclose(y[1], [0, math.cos(0.03), 0, math.sin(0.03), 0], atol=1e-15)
    np.testing.assert_allclose(y[2], [-math.sin(3), 0, math.cos(3), 0, 0], atol=1e-15)
    np.testing.assert_allclose(y[3], [0, -math.sin(0.03), 0, math.cos(0.03), 0], atol=1e-15)
    np.testing.assert_array_equal(y[4], [0, 0, 0, 0, 1])
    np.testing.assert_array_equal(O.rope_neox(e, 0, 4, 10000.0), e)


def test_rope_scores_depend_on_relative_position_only():
    """<RoPE(q, m), RoPE(k, n)> = <RoPE(q, m - n), k>, and norms are kept."""
    rng = np.random.default_rng(13)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    for m, n in ((5, 2), (1000, 997), (37, 40), (32767, 0)):
        lhs = O.rope_neox(q, m, 64, 10000.0) @ O.rope_neox(k, n, 64, 10000.0)
        rhs = O.rope_neox(q, m - n, 64, 10000.0) @ k
        assert abs(lhs - rhs) < 1e-9
    assert abs(np.linalg.norm(O.rope_neox(q, 777, 64, 10000.0)) - np.linalg.norm(q)) < 1e-12


def test_sylvester_hadamard_matches_scipy_and_is_orthonormal():
    """The Sylvester construction equals scipy's Hadamard matrix, has entries
    (-1)^popcount(i & j), and H/sqrt(D) keeps norms and every dot product
    (ik_llama.cpp #2045: the rotation leaves q.k unchanged)."""
    for D in (1, 2, 4, 32, 64, 128):
        H = O.sylvester_hadamard(D)
        assert np.array_equal(H, scipy.linalg.hadamard(D))
        assert np.array_equal(H @ H.T, D * np.eye(D))
    H = O.sylvester_hadamard(128)
    i, j = np.meshgrid(np.arange(128), np.arange(128), indexing="ij")
    parity = np.vectorize(lambda v: bin(v).count("1") & 1)(i & j)
    assert np.array_equal(H, 1 - 2 * parity)
    rng = np.random.default_rng(14)
    x, y = rng.standard_normal((2, 128))
    hx, hy = O.hadamard_rotate(x), O.hadamard_rotate(y)
    assert abs(hx @ hy - x @ y) < 1e-12 and abs(np.linalg.norm(hx) - np.linalg.norm(x)) < 1e-12
    with pytest.raises(ValueError):
        O.sylvester_hadamard(48)
    # worked by hand: H_4 (1, 2, 3, 4) = (10, -2, -4, 0), and the orthonormal rotation halves it
    assert O.hadamard_rotate(np.array([1.0, 2.0, 3.0, 4.0])).tolist() == [5.0, -1.0, -2.0, 0.0]
    assert O.hadamard_rotate(np.array([[0.0, 0.0, 0.0, 2.0]])).tolist() == [[1.0, -1.0, -1.0, 1.0]]


def _rot_inputs(seed=15):
    rng = np.random.default_rng(seed)
    xk = rng.standard_normal((3, 1, 128)) * 2 + 0.5
    xq = rng.standard_normal((3, 4, 128))
    ln_w = 1 + 0.1 * rng.standard_normal(128)
    ln_b = 0.1 * rng.standard_normal(128)
    pos = np.array([5, 100, 4000])
    return xk, xq, ln_w, ln_b, pos


def test_cached_key_moves_by_unrotate_rope_delta_rerotate():
    """ik_llama.cpp #2063 (K-shift commit): the cached key is
    H*concat(RoPE(k_pe, p), k_nope); moving it to position p + d is un-Hadamard
    (H orthonormal and symmetric), a RoPE by d of the pe part, and re-Hadamard."""
    xk, _, ln_w, ln_b, pos = _rot_inputs()
    d = 37
    cached = O.index_rotate(xk, pos, 64, 10000.0, ln_w, ln_b, 1e-6, layer_norm_first=True)
    Hn = O.sylvester_hadamard(128) / math.sqrt(128)
    moved = np.stack([O.rope_neox(cached[r] @ Hn, d, 64, 10000.0) @ Hn for r in range(3)])
    direct = O.index_rotate(xk, pos + d, 64, 10000.0, ln_w, ln_b, 1e-6, layer_norm_first=True)
    np.testing.assert_allclose(moved, direct, atol=1e-12)


def test_key_layer_norm_comes_before_rope():
    """Without the rotation, the nope part of a prepared key is the LayerNorm of
    the whole input row (torch's layer_norm), untouched by RoPE; the pe part is
    that LayerNorm turned by RoPE."""
    xk, _, ln_w, ln_b, pos = _rot_inputs()
    got = O.index_rotate(xk, pos, 64, 10000.0, ln_w, ln_b, 1e-6, layer_norm_first=True, hadamard=False)
    ln = torch.nn.functional.layer_norm(torch.tensor(xk), (128,), torch.tensor(ln_w), torch.tensor(ln_b),
                                        1e-6).numpy()
    np.testing.assert_allclose(got[..., 64:], ln[..., 64:], atol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(got[..., :64], axis=-1), np.linalg.norm(ln[..., :64], axis=-1),
                               atol=1e-12)


def test_rotated_queries_and_keys_give_the_same_scores():
    """The Hadamard rotation changes no index score (ik_llama.cpp #2045)."""
    xk, xq, ln_w, ln_b, pos = _rot_inputs()
    w = np.array([0.5, -1.0, 2.0, 0.25])
    kr = O.index_rotate(xk, pos, 64, 10000.0, ln_w, ln_b, 1e-6, layer_norm_first=True)[:, 0]
    kp = O.index_rotate(xk, pos, 64, 10000.0, ln_w, ln_b, 1e-6, layer_norm_first=True, hadamard=False)[:, 0]
    for r in range(3):
        qr = O.index_rotate(xq[r:r + 1], pos[r:r + 1], 64, 10000.0)[0]
        qp = O.index_rotate(xq[r:r + 1], pos[r:r + 1], 64, 10000.0, hadamard=False)[0]
        np.testing.assert_allclose(O.index_scores_row(qr, kr, w, 0.1), O.index_scores_row(qp, kp, w, 0.1),
                                   atol=1e-12)


# ------------------------------------------- P14 FP8 (e4m3) indexer operands
def test_e4m3_grid_is_the_format_and_decodes_like_torch():
    """127 non-negative finite values: subnormal step 2^-9, smallest normal 2^-6, eight values per binade,
    largest 448; code i decodes (torch's float8_e4m3fn) to the i-th value."""
    g = O.e4m3_grid()
    assert g.size == 127 and g[0] == 0 and g[1] == 2.0 ** -9 and g[8] == 2.0 ** -6 and g[-1] == 448.0
    for e in range(1, 15):
        binade = g[8 * e: 8 * e + 8]
        assert np.array_equal(binade, 2.0 ** (e - 7) * (1 + np.arange(8) / 8))
    decoded = torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(decoded, g)


def test_e4m3_rounding_ties_to_even_and_matches_torch():
    hand = {1.0625: 1.0, 1.1875: 1.25, 2.0 ** -10: 0.0, 3 * 2.0 ** -11: 2.0 ** -9, 463.9: 448.0, -1.0625: -1.0,
            0.3: 0.3125, 17.0: 16.0, 19.0: 20.0}
    got = O.e4m3_round(np.array(list(hand)))
    assert got.tolist() == list(hand.values())
    rng = np.random.default_rng(16)
    y = np.concatenate([rng.uniform(-463, 463, 50000), rng.uniform(-0.03, 0.03, 20000),
                        O.e4m3_grid()[1:-1] + np.diff(O.e4m3_grid())[1:] / 2])   # exact midpoints
    y = y.astype(np.float32).astype(np.float64)
    ref = torch.tensor(y, dtype=torch.float32).to(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(O.e4m3_round(y), ref)
    with pytest.raises(ValueError):
        O.e4m3_round(np.array([464.0]))


def test_fp8_quantization_maps_each_vector_amax_to_448_within_the_grid_error():
    rng = np.random.default_rng(17)
    x = rng.standard_normal((6, 5, 128)) * rng.choice([1e-3, 1.0, 50.0], (6, 5, 1))
    x[2, 3] = 0.0
    codes, sc = O.fp8_quantize(x)
    amax = np.abs(x).max(axis=-1)
    nz = amax > 0
    assert np.array_equal(np.abs(codes).max(axis=-1)[nz], np.full(nz.sum(), 448.0))
    assert np.all(codes[2, 3] == 0) and sc[2, 3] == 1.0
    assert np.all(np.isin(np.abs(codes), O.e4m3_grid()))
    # half a grid step: 2^-4 of the value in the normal range, 2^-10 * scale below it (plus fp32 inputs)
    err = np.abs(codes * sc[..., None] - x)
    bound = 2.0 ** -4 * np.abs(x) + 2.0 ** -10 * sc[..., None] + 1e-6 * amax[..., None]
    assert np.all(err <= bound)


def test_fp8_scores_equal_plain_scores_when_the_operands_are_e4m3_values_with_amax_448():
    """Unit scales and representable operands make the quantisation exact, so the FP8 score is the plain one."""
    rng = np.random.default_rng(18)
    g = O.e4m3_grid()
    q = rng.choice(g, (4, 32)) * rng.choice([-1, 1], (4, 32))
    k = rng.choice(g, (9, 32)) * rng.choice([-1, 1], (9, 32))
    q[:, 0] = 448.0
    k[:, 5] = -448.0
    w = np.array([0.5, -1.0, 2.0, 0.25])
    assert np.array_equal(O.index_scores_fp8_row(q, k, w, 1 / 64), O.index_scores_row(q, k, w, 1 / 64))
    # a per-vector factor of 2 changes scales only, not codes: the score doubles per factor
    assert np.array_equal(O.index_scores_fp8_row(2 * q, k, w, 1 / 64), 2 * O.index_scores_row(q, k, w, 1 / 64))
    assert np.array_equal(O.index_scores_fp8_row(q, 4 * k, w, 1 / 64), 4 * O.index_scores_row(q, k, w, 1 / 64))


# ------------------------------------------- planted mistakes are caught
def _run_pins():
    failures = 0
    for fn in (test_hand_index_scores_and_topk, test_hand_attend_sets, test_softmax_two_key_closed_form,
               test_topk_matches_brute_force_with_ties, test_walsh_hadamard_rotation_leaves_scores_unchanged,
               test_expand_selection_examples, test_pooling_starts_at_first_valid_token_and_drops_partial_pool,
               lambda: test_topk_covering_all_keys_equals_dense_attention(1),
               test_absorbed_mla_equals_literal_expand_kv, test_rope_neox_pairs_halves_with_closed_form_angles,
               test_rope_scores_depend_on_relative_position_only,
               test_sylvester_hadamard_matches_scipy_and_is_orthonormal,
               test_cached_key_moves_by_unrotate_rope_delta_rerotate, test_key_layer_norm_comes_before_rope,
               test_rotated_queries_and_keys_give_the_same_scores, test_e4m3_grid_is_the_format_and_decodes_like_torch,
               test_e4m3_rounding_ties_to_even_and_matches_torch,
               test_fp8_quantization_maps_each_vector_amax_to_448_within_the_grid_error,
               test_fp8_scores_equal_plain_scores_when_the_operands_are_e4m3_values_with_amax_448,
               test_pool_topk_matches_brute_force_over_fully_visible_pools):
        try:
            fn()
        except (AssertionError, ValueError, IndexError):
            failures += 1
    return failures


@pytest.mark.parametrize("mutant", ["scale_outside_relu_negated", "drop_weight", "tie_largest_index",
                                    "no_dedupe", "softmax_no_max_shift_sign", "pool_from_zero",
                                    "tail_off_by_one", "absorb_transposed", "rope_adjacent_pairs",
                                    "rope_frequency_exponent", "hadamard_before_rope", "layer_norm_after_rope",
                                    "hadamard_unnormalised", "e4m3_ties_away", "e4m3_two_mantissa_bits",
                                    "fp8_key_scale_dropped", "pool_visible_at_first_token"])
def test_pins_catch_planted_mistakes(monkeypatch, mutant):
    """Plant a plausible mistake in the oracle (on the CPU) and check a pin fails."""
    assert _run_pins() == 0
    if mutant == "scale_outside_relu_negated":
        orig = O.index_scores_row
        monkeypatch.setattr(O, "index_scores_row",
                            lambda q, k, w, s: orig(q, k, w, -s) * -1.0)
    elif mutant == "drop_weight":
        monkeypatch.setattr(O, "index_scores_row",
                            lambda q, k, w, s: np.maximum(0, s * (O.f64(q) @ O.f64(k).T)).sum(0))
    elif mutant == "tie_largest_index":
        def bad(cand, sc, k):
            cand = np.asarray(cand); sc = np.asarray(sc, float)
            order = np.lexsort((-cand, -sc))
            out = np.full(k, -1); n = min(k, cand.size); out[:n] = cand[order[:n]]
            return out
        monkeypatch.setattr(O, "topk_row", bad)
    elif mutant == "no_dedupe":
        monkeypatch.setattr(O, "index_set",
                            lambda row, n: np.array([i for i in O.i64(row).tolist() if 0 <= i < n], dtype=np.int64))
    elif mutant == "softmax_no_max_shift_sign":
        def bad_attend(q, k, v, scale):
            k = O.f64(k); v = O.f64(v)
            z = -scale * (k @ O.f64(q)); p = np.exp(z - z.max())
            return (p @ v) / p.sum(), float(z.max() + math.log(p.sum()))
        monkeypatch.setattr(O, "attend_row", bad_attend)
    elif mutant == "pool_from_zero":
        orig = O.pool_states
        monkeypatch.setattr(O, "pool_states", lambda k, g, f, L, kp, w, b, e: orig(k, g, 0, L - f, kp, w, b, e))
    elif mutant == "tail_off_by_one":
        orig = O.expand_selection
        def bad(pools, t, f, L, kp, npools, width):
            return orig(pools, t - 1, f, L, kp, npools, width) if t > f else orig(pools, t, f, L, kp, npools, width)
        monkeypatch.setattr(O, "expand_selection", bad)
    elif mutant == "absorb_transposed":
        orig = O.mla_absorbed_row
        def bad2(q, lat, uk, uv, row, scale):
            out, lse = orig(q, lat, uk, uv, row, scale)
            return out[::-1].copy(), lse[::-1].copy()
        monkeypatch.setattr(O, "mla_absorbed_row", bad2)
    elif mutant == "rope_adjacent_pairs":
        def gptj(x, pos, n_rope, theta):
            x = O.f64(x).copy()
            for i in range(n_rope // 2):
                ang = pos * theta ** (-2.0 * i / n_rope)
                a, b = x[..., 2 * i].copy(), x[..., 2 * i + 1].copy()
                x[..., 2 * i] = a * math.cos(ang) - b * math.sin(ang)
                x[..., 2 * i + 1] = b * math.cos(ang) + a * math.sin(ang)
            return x
        monkeypatch.setattr(O, "rope_neox", gptj)
    elif mutant == "rope_frequency_exponent":
        orig_rope = O.rope_neox
        def bad_freq(x, pos, n_rope, theta):
            x = O.f64(x).copy()
            half = n_rope // 2
            for i in range(half):
                ang = pos * theta ** (-1.0 * i / n_rope)
                a, b = x[..., i].copy(), x[..., i + half].copy()
                x[..., i] = a * math.cos(ang) - b * math.sin(ang)
                x[..., i + half] = b * math.cos(ang) + a * math.sin(ang)
            return x
        monkeypatch.setattr(O, "rope_neox", bad_freq)
    elif mutant in ("hadamard_before_rope", "layer_norm_after_rope"):
        def bad_rotate(x, pos, n_rope, theta, ln_w=None, ln_b=None, eps=1e-6, layer_norm_first=False,
                       hadamard=True):
            x = O.f64(x)
            out = np.empty_like(x)
            for r in range(x.shape[0]):
                y = x[r]
                if mutant == "hadamard_before_rope":
                    if layer_norm_first:
                        y = O.layer_norm(y, ln_w, ln_b, eps)
                    if hadamard:
                        y = O.hadamard_rotate(y)
                    y = O.rope_neox(y, int(pos[r]), n_rope, theta)
                else:
                    y = O.rope_neox(y, int(pos[r]), n_rope, theta)
                    if layer_norm_first:
                        y = O.layer_norm(y, ln_w, ln_b, eps)
                    if hadamard:
                        y = O.hadamard_rotate(y)
                out[r] = y
            return out
        monkeypatch.setattr(O, "index_rotate", bad_rotate)
    elif mutant == "hadamard_unnormalised":
        monkeypatch.setattr(O, "hadamard_rotate", lambda x: O.f64(x) @ O.sylvester_hadamard(O.f64(x).shape[-1]).T)
    elif mutant == "e4m3_ties_away":
        orig_round = O.e4m3_round
        def away(y):
            y = O.f64(y)
            a = np.abs(y)
            g = O.e4m3_grid()
            hi = np.clip(np.searchsorted(g, a), 1, g.size - 1)
            q = np.where(g[hi] - a <= a - g[hi - 1], g[hi], g[hi - 1])
            return np.copysign(q, y)
        monkeypatch.setattr(O, "e4m3_round", away)
    elif mutant == "e4m3_two_mantissa_bits":
        def grid2():
            vals = [m * 2.0 ** -8 for m in range(4)]
            for e in range(1, 16):
                for m in range(4):
                    vals.append(2.0 ** (e - 7) * (1 + m / 4))
            return np.array(vals)
        monkeypatch.setattr(O, "e4m3_grid", grid2)
    elif mutant == "fp8_key_scale_dropped":
        def no_kscale(q_row, keys, w_row, scale):
            qc, qs = O.fp8_quantize(q_row)
            kc, ks = O.fp8_quantize(keys)
            act = np.maximum(0.0, float(scale) * qs[:, None] * (qc @ kc.T))
            return (O.f64(w_row)[:, None] * act).sum(axis=0) + 0.0
        monkeypatch.setattr(O, "index_scores_fp8_row", no_kscale)
    elif mutant == "pool_visible_at_first_token":
        # a pool counted visible once its first token is, instead of all of its tokens
        def early(q_pos, kv_start, n_pools, kpool):
            f = int(kv_start)
            if q_pos < f:
                return np.zeros(0, dtype=np.int64)
            return np.arange(0, min((int(q_pos) - f) // kpool + 1, int(n_pools)), dtype=np.int64)
        monkeypatch.setattr(O, "visible_pools", early)
    assert _run_pins() > 0, f"mutant {mutant} survived every pin"
