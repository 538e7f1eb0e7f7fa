"""CPU oracle for the DSA layer: plain, slow, f64.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this
module: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline / reference arm call it.  It shares no code with the CUDA library
(``sparse_attention_sum_b200``); the two meet only in the seeded input
generators of ``workloads``.

Every value is read as the exact bf16 / fp32 number and converted to float64
before any arithmetic.  A library primitive (matrix product, sort, exp) may
serve as one step; nothing is blocked, fused or reordered beyond what the
definitions say, so each function can be checked against the pages by eye.

Sources (web pages on DeepSeek Sparse Attention):

* [fak-sparse]  fak note "GLM-5.2: the DSA sparse attention moves onto the
  pure fak kernel (2026-06-23)".
* [ik-2063]     ik_llama.cpp pull request #2063 "Another DSA attempt", with the
  squashed commit messages of PR #2045.
* [metrale]     docs.metrale.ai, module ``glm5next_dsa_ref`` (CPU reference for
  the GLM-5.3-Flash kpool indexer and NoPE MLA): function list and invariants.

Conventions (readings where the pages leave a step open are marked READING):

* A query row is identified by its batch index ``b`` and its absolute
  position ``q_pos``.  Keys are absolute cache rows ``s`` of batch ``b``.
* ``kv_start[b]`` is the first valid (non-padding) key row, ``kv_len[b]`` one
  past the last valid row.
* ``INVALID = -1`` fills every index slot that holds no token ([metrale],
  constant ``INVALID`` and the ``expand_selection`` invariant).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
except the exact order of the ``expand_selection`` output beyond the pages'
worked examples (see the ``expand_selection`` docstring): parity unpinned for
that ordering choice.
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np

try:  # torch is only used to read bf16 tensors exactly
    import torch
except Exception:  # pragma: no cover
    torch = None

INVALID = -1


# ---------------------------------------------------------------------------
# exact conversion
# ---------------------------------------------------------------------------
def f64(x) -> np.ndarray:
    """Exact float64 copy of a torch tensor (fp32 / bf16) or array-like."""
    if torch is not None and isinstance(x, torch.Tensor):
        return x.detach().to(torch.float64).cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def i64(x) -> np.ndarray:
    if torch is not None and isinstance(x, torch.Tensor):
        return x.detach().cpu().numpy().astype(np.int64)
    return np.asarray(x, dtype=np.int64)


# ---------------------------------------------------------------------------
# S1: visibility
# ---------------------------------------------------------------------------
def visible_keys(q_pos: int, kv_start: int, kv_len: int) -> np.ndarray:
    """Key rows a query at absolute position ``q_pos`` may see.

    [metrale] ``visible``: causal and not padding.  READING: the causal
    diagonal is inclusive (a query sees its own key, as in the llama KQ mask
    and in decode where the new token's key is already cached, [ik-2063]
    "+ base causal mask"), and visibility never crosses sequences ([ik-2063]
    UPDATE 5: cross-sequence keys are driven to -inf).  A query with
    ``q_pos < kv_start`` is a padded row and sees nothing.
    """
    hi = min(int(q_pos), int(kv_len) - 1)
    lo = int(kv_start)
    if hi < lo:
        return np.zeros(0, dtype=np.int64)
    return np.arange(lo, hi + 1, dtype=np.int64)


def visible_pools(q_pos: int, kv_start: int, n_pools: int, kpool: int) -> np.ndarray:
    """Pools a query at ``q_pos`` may see (kpool variant).

    [metrale] invariants: pooling starts at the first valid token and a pool
    is valid only if all ``kpool`` slots are valid.  READING: pool ``p``
    (tokens ``kv_start + p*kpool ... kv_start + p*kpool + kpool - 1``) is
    visible when its last token is causally visible.
    """
    f = int(kv_start)
    if q_pos < f:
        return np.zeros(0, dtype=np.int64)
    n_vis = min((int(q_pos) - f + 1) // kpool, int(n_pools))
    return np.arange(0, n_vis, dtype=np.int64)


# ---------------------------------------------------------------------------
# S2: lightning-indexer scores
# ---------------------------------------------------------------------------
def index_scores_row(q_row, keys, w_row, scale: float) -> np.ndarray:
    """``I[s] = sum_h w[h] * relu(scale * q[h] . k[s])`` for the given key rows.

    [fak-sparse] section 3 (learned-index score dots ``sum_h
    weights[h]*relu(scale*dot(q_h, key))``, computed in f64 on the host) and
    [metrale] ``index_scores``.  ``q_row`` is ``[H_I, D_I]``, ``keys`` is
    ``[n, D_I]`` (one shared MQA key per token), ``w_row`` is ``[H_I]``.
    A signed zero result is returned as +0.
    """
    q = f64(q_row)
    k = f64(keys)
    w = f64(w_row)
    dots = q @ k.T                                   # [H_I, n]
    per_head = np.maximum(0.0, scale * dots)         # relu(scale * q.k)
    out = (w[:, None] * per_head).sum(axis=0)        # sum over heads
    return out + 0.0                                 # -0.0 -> +0.0


def index_scores(q_idx, k_idx, w, scale: float, q_pos, kv_start, kv_len,
                 rows: Optional[Iterable[Tuple[int, int]]] = None) -> np.ndarray:
    """Dense score matrix ``[B, n_q, n_kv]`` with ``-inf`` where not visible.

    ``rows`` restricts the work to the listed ``(b, t)`` rows (others stay
    ``-inf``).  Only meant for small problems or sampled rows.
    """
    B, T = q_idx.shape[0], q_idx.shape[1]
    S = k_idx.shape[1]
    qp, ks, kl = i64(q_pos), i64(kv_start), i64(kv_len)
    out = np.full((B, T, S), -np.inf)
    it = rows if rows is not None else ((b, t) for b in range(B) for t in range(T))
    for b, t in it:
        cand = visible_keys(qp[b, t], ks[b], kl[b])
        if cand.size:
            out[b, t, cand] = index_scores_row(q_idx[b, t], k_idx[b][cand], w[b, t], scale)
    return out


# ---------------------------------------------------------------------------
# S3: deterministic top-k
# ---------------------------------------------------------------------------
def topk_row(cand: np.ndarray, cand_scores: np.ndarray, k: int) -> np.ndarray:
    """Top ``k`` of the candidates, ordered by higher score then smaller index.

    [metrale] ``topk_pools``: ordered by higher score, then smaller index, so
    ties resolve the same way on every run; [ik-2063] ``ggml_top_k(min(top_k,
    n_tokens))``.  READING: with fewer than ``k`` candidates all are emitted and
    the row is padded with INVALID; output is in rank order.
    """
    cand = np.asarray(cand, dtype=np.int64)
    sc = np.asarray(cand_scores, dtype=np.float64) + 0.0
    order = np.lexsort((cand, -sc))                  # primary: -score, then index
    n = min(int(k), cand.size)
    out = np.full(int(k), INVALID, dtype=np.int64)
    out[:n] = cand[order[:n]]
    return out


def topk(scores: np.ndarray, k: int, q_pos, kv_start, kv_len) -> np.ndarray:
    """Row-wise top-k over the visible keys of a dense score matrix ``[B, T, S]``."""
    B, T, _ = scores.shape
    qp, ks, kl = i64(q_pos), i64(kv_start), i64(kv_len)
    out = np.full((B, T, int(k)), INVALID, dtype=np.int64)
    for b in range(B):
        for t in range(T):
            cand = visible_keys(qp[b, t], ks[b], kl[b])
            out[b, t] = topk_row(cand, scores[b, t, cand], k)
    return out


# ---------------------------------------------------------------------------
# S4: sparse attention over the selected keys
# ---------------------------------------------------------------------------
def index_set(idx_row, n_kv: int) -> np.ndarray:
    """The key set an index row denotes.

    [metrale] ``topk_to_mask``: duplicate indices collapse (a repeated token
    is attended once); out-of-range and INVALID entries are dropped.  The set
    is listed in order of first appearance.
    """
    seen = set()
    keep = []
    for i in i64(idx_row).tolist():
        if 0 <= i < n_kv and i not in seen:
            seen.add(i)
            keep.append(i)
    return np.asarray(keep, dtype=np.int64)


def attend_row(q_row, k_rows, v_rows, scale: float) -> Tuple[np.ndarray, float]:
    """One head of softmax attention over an explicit key list.

    [fak-sparse] "What changed": the host loop is dot*scale, softmax in place,
    then the in-order weighted sum of V; the key width may differ from the
    value width.  ``q_row`` is ``[kd]``, ``k_rows`` ``[n, kd]``, ``v_rows``
    ``[n, vd]``.  Returns ``(o[vd], lse)``; READING: an empty key list gives
    ``o = 0`` and ``lse = -inf``.
    """
    k = f64(k_rows)
    v = f64(v_rows)
    if k.shape[0] == 0:
        return np.zeros(v.shape[1]), -math.inf
    z = scale * (k @ f64(q_row))                     # dot * scale
    m = z.max()
    p = np.exp(z - m)                                # softmax numerators
    denom = p.sum()
    o = p @ v                                        # sum of p_i V_i
    return o / denom, float(m + math.log(denom))


def sparse_attend_row(q_bt, k_cache_b, v_cache_b, idx_row, scale: float):
    """All heads of one query row.

    ``q_bt`` is ``[H, kd]``; ``k_cache_b`` is ``[n_kv, Hk, kd]`` and
    ``v_cache_b`` ``[n_kv, Hk, vd]`` with ``Hk`` dividing ``H`` (``Hk = 1`` is the
    shared MLA latent, [fak-sparse] MLA key/value widths).  Head ``h`` reads
    KV head ``h // (H // Hk)``.  Returns ``(out[H, vd], lse[H])``.
    """
    H = q_bt.shape[0]
    n_kv, Hk = k_cache_b.shape[0], k_cache_b.shape[1]
    U = index_set(idx_row, n_kv)
    vd = v_cache_b.shape[2]
    out = np.zeros((H, vd))
    lse = np.full(H, -math.inf)
    if U.size == 0:
        return out, lse
    if Hk == 1:
        # shared latent: the same key/value rows for every head, as one product
        kU = f64(k_cache_b[U, 0])                    # [n, kd]
        vU = f64(v_cache_b[U, 0])                    # [n, vd]
        z = scale * (f64(q_bt) @ kU.T)               # [H, n]
        m = z.max(axis=1, keepdims=True)
        p = np.exp(z - m)
        denom = p.sum(axis=1, keepdims=True)
        return (p @ vU) / denom, (m + np.log(denom))[:, 0]
    for h in range(H):
        hk = h // (H // Hk)
        out[h], lse[h] = attend_row(q_bt[h], k_cache_b[U, hk], v_cache_b[U, hk], scale)
    return out, lse


def sparse_attend(q, k_cache, v_cache, idx, scale: float,
                  rows: Optional[Iterable[Tuple[int, int]]] = None):
    """``out[B, T, H, vd]`` and ``lse[B, T, H]`` for the listed (or all) rows."""
    B, T, H = q.shape[0], q.shape[1], q.shape[2]
    vd = v_cache.shape[-1]
    out = np.zeros((B, T, H, vd))
    lse = np.full((B, T, H), -math.inf)
    it = rows if rows is not None else ((b, t) for b in range(B) for t in range(T))
    for b, t in it:
        out[b, t], lse[b, t] = sparse_attend_row(q[b, t], k_cache[b], v_cache[b], idx[b, t], scale)
    return out, lse


# ---------------------------------------------------------------------------
# S5: the layer (indexer -> top-k -> sparse attention)
# ---------------------------------------------------------------------------
def layer_row(b: int, t: int, wl_t, top_k: int, idx_scale: float, attn_scale: float,
              q, k_cache, v_cache):
    """One query row of the whole DSA layer; returns ``(idx, out, lse, scores)``.

    [fak-sparse] sections "The selection stays host-side" and 3: index-score
    dots and top-k pick the keys, then the sparse attend runs over them.
    ``wl_t`` is a dict with ``q_idx, k_idx, w, q_pos, kv_start, kv_len``.
    """
    qp = int(i64(wl_t["q_pos"])[b, t])
    ks = int(i64(wl_t["kv_start"])[b])
    kl = int(i64(wl_t["kv_len"])[b])
    cand = visible_keys(qp, ks, kl)
    sc = index_scores_row(wl_t["q_idx"][b, t], wl_t["k_idx"][b][cand], wl_t["w"][b, t], idx_scale) \
        if cand.size else np.zeros(0)
    sel = topk_row(cand, sc, top_k)
    out, lse = sparse_attend_row(f64(q[b, t]), k_cache[b], v_cache[b], sel, attn_scale)
    return sel, out, lse, (cand, sc)


def dense_causal_attend(q, k_cache, v_cache, scale: float, q_pos, kv_start, kv_len):
    """Textbook masked softmax attention over every visible key.

    Written independently of :func:`sparse_attend` (full score matrix, row
    softmax) so that the "top_k >= visible tokens equals dense attention"
    property of [ik-2063] (PPL byte-identical to the dense baseline when
    ``top_k >= n_tokens``) can pin the sparse path.
    """
    q = f64(q)
    k = f64(k_cache)
    v = f64(v_cache)
    B, T, H, _ = q.shape
    S, Hk = k.shape[1], k.shape[2]
    qp, ks, kl = i64(q_pos), i64(kv_start), i64(kv_len)
    out = np.zeros((B, T, H, v.shape[-1]))
    pos = np.arange(S)
    for b in range(B):
        for h in range(H):
            hk = h // (H // Hk)
            logits = scale * np.einsum("td,sd->ts", q[b, :, h], k[b, :, hk])
            mask = (pos[None, :] >= ks[b]) & (pos[None, :] <= qp[b][:, None]) & (pos[None, :] < kl[b])
            logits = np.where(mask, logits, -np.inf)
            rowmax = np.max(np.where(mask, logits, -np.inf), axis=1, keepdims=True)
            rowmax = np.where(np.isfinite(rowmax), rowmax, 0.0)
            e = np.where(mask, np.exp(logits - rowmax), 0.0)
            den = e.sum(axis=1, keepdims=True)
            den = np.where(den > 0, den, 1.0)
            out[b, :, h] = (e / den) @ v[b, :, hk]
    return out


# ---------------------------------------------------------------------------
# S6: kpool LayerNorm + pooling
# ---------------------------------------------------------------------------
def layer_norm(x, w, b, eps: float) -> np.ndarray:
    """LayerNorm over the last axis: subtract the mean, divide by the standard
    deviation, then ``w * x + b`` ([metrale] ``layer_norm``; k_norm has a bias).

    READING: the variance is the biased (population) variance and ``eps`` is
    added inside the square root, as in torch's LayerNorm; ``eps`` must be
    positive ([ik-2063]: eps 0 aborts ggml_norm; the GGUF port mirrors 1e-5,
    the HF reference uses 1e-6).
    """
    if not eps > 0:
        raise ValueError("layer_norm eps must be > 0")
    x = f64(x)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mu) / np.sqrt(var + eps)
    if w is not None:
        y = y * f64(w)
    if b is not None:
        y = y + f64(b)
    return y


def n_pools_of(kv_start: int, kv_len: int, kpool: int) -> int:
    """Number of complete pools: a trailing partial pool is not a pool."""
    return max(0, (int(kv_len) - int(kv_start)) // int(kpool))


def pool_states(k, gate, kv_start: int, kv_len: int, kpool: int, ln_w, ln_b, eps: float):
    """Pooled indexer keys of one sequence: ``[n_pools, D]``.

    [metrale] ``pool_states`` and invariants: the pool softmax runs over the
    slot axis, separately for each channel; pooling starts at the first valid
    token (left padding ``[P,P,A,B,C,D]`` gives pool 0 = ``[A,B,C,D]``); a
    trailing partial pool is not a pool.  READING: k_norm (LayerNorm with bias)
    is applied to each token's key before pooling, since it is part of the
    indexer key.
    """
    k = f64(k)
    g = f64(gate)
    f = int(kv_start)
    P = n_pools_of(f, kv_len, kpool)
    D = k.shape[-1]
    out = np.zeros((P, D))
    for p in range(P):
        rows = f + p * kpool + np.arange(kpool)
        kn = layer_norm(k[rows], ln_w, ln_b, eps)            # [kpool, D]
        gs = g[rows]                                         # [kpool, D]
        e = np.exp(gs - gs.max(axis=0, keepdims=True))       # softmax over slots,
        sm = e / e.sum(axis=0, keepdims=True)                # per channel
        out[p] = (sm * kn).sum(axis=0)
    return out


def kept_pools(kv_start: int, kv_len: int, kpool: int) -> np.ndarray:
    """Ids of the pools ``pool_states`` keeps, from padding and length alone.

    [metrale] ``kept_pools``.  READING: ids are counted in the frame that
    starts at the first valid token, so they are ``0 .. n_pools-1``.
    """
    return np.arange(n_pools_of(kv_start, kv_len, kpool), dtype=np.int64)


# ---------------------------------------------------------------------------
# S7: pool selection and expand_selection
# ---------------------------------------------------------------------------
def topk_pools_row(q_row, pooled, w_row, scale: float, q_pos: int, kv_start: int,
                   n_pools: int, kpool: int, select_k: int):
    """Index scores over the visible pools, then the deterministic top-k.

    [metrale] ``index_scores`` (per query, per pool) and ``topk_pools``:
    invalid candidates score ``f32::MIN`` and so are never chosen ahead of a
    valid one; READING: they are never emitted at all (the row is padded with
    INVALID instead), matching ``expand_selection``'s INVALID fill.
    """
    cand = visible_pools(q_pos, kv_start, n_pools, kpool)
    sc = index_scores_row(q_row, f64(pooled)[cand], w_row, scale) if cand.size else np.zeros(0)
    return topk_row(cand, sc, select_k), (cand, sc)


def expand_selection(pool_row, q_pos: int, kv_start: int, kv_len: int, kpool: int,
                     n_pools: int, out_width: int) -> np.ndarray:
    """Selected pools -> raw token indices, then the visible tail, then INVALID.

    [metrale] ``expand_selection``: every row is written for all ``out_width``
    entries; the output starts filled with INVALID and a padded query row stays
    that way.  The invariants say the tail append covers the trailing partial
    pool.  READINGS (parity unpinned beyond the pages' examples): pools are
    expanded in rank order with their ``kpool`` tokens ascending; the tail is
    every visible token after the last fully visible pool, ascending.
    """
    out = np.full(int(out_width), INVALID, dtype=np.int64)
    f = int(kv_start)
    if q_pos < f:
        return out
    pos = 0
    for p in i64(pool_row).tolist():
        if p < 0 or p >= int(n_pools):         # INVALID and out-of-range ids hold no pool
            continue
        for j in range(kpool):
            out[pos] = f + p * kpool + j
            pos += 1
    n_vis = min((int(q_pos) - f + 1) // kpool, int(n_pools))
    last = min(int(q_pos), int(kv_len) - 1)
    for s in range(f + n_vis * kpool, last + 1):
        out[pos] = s
        pos += 1
    return out


# ---------------------------------------------------------------------------
# S8: NoPE MLA (literal expand_kv form, and the absorbed form)
# ---------------------------------------------------------------------------
def linear(x, w) -> np.ndarray:
    """``y = x @ w^T`` for ``x [m, k]`` and ``w [n, k]`` ([metrale] ``linear``)."""
    return f64(x) @ f64(w).T


def expand_kv(latent_rows, w_uk, w_uv):
    """Per-head K and V from the compressed latent ([metrale] ``expand_kv``).

    NoPE only (no rope section), so K is exactly the q/k head width.
    ``latent_rows`` is ``[n, L]``; ``w_uk``/``w_uv`` are ``[H, d, L]``.  Returns
    ``K [n, H, d]`` and ``V [n, H, dv]``.
    """
    c = f64(latent_rows)
    uk = f64(w_uk)
    uv = f64(w_uv)
    H = uk.shape[0]
    K = np.stack([linear(c, uk[h]) for h in range(H)], axis=1)
    V = np.stack([linear(c, uv[h]) for h in range(H)], axis=1)
    return K, V


def mla_masked_attention_row(q_bt, latent_b, w_uk, w_uv, tok_row, scale: float):
    """[metrale] ``mla_masked_attention``: NoPE MLA of one query row over its
    selected token set, computed literally (expand the selected latent rows to
    per-head K/V, then per-head softmax attention).  ``q_bt`` is ``[H, d]``.
    Returns ``(out[H, dv], lse[H])``.
    """
    n_kv = latent_b.shape[0]
    U = index_set(tok_row, n_kv)
    H = q_bt.shape[0]
    dv = w_uv.shape[1]
    if U.size == 0:
        return np.zeros((H, dv)), np.full(H, -math.inf)
    K, V = expand_kv(f64(latent_b[U]), w_uk, w_uv)           # [n, H, d]
    out = np.zeros((H, dv))
    lse = np.zeros(H)
    for h in range(H):
        out[h], lse[h] = attend_row(f64(q_bt[h]), K[:, h], V[:, h], scale)
    return out, lse


def mla_absorbed_row(q_bt, latent_b, w_uk, w_uv, tok_row, scale: float):
    """The same NoPE MLA row in absorbed form, for the absorption identity.

    ``q~_h = W_UK,h^T q_h`` (so ``q_h . (W_UK,h c) = q~_h . c``), attention over
    the latent rows themselves, then ``o_h = W_UV,h o~_h``.  Written as a
    separate routine so the algebraic identity can be checked in f64.
    """
    uk = f64(w_uk)
    uv = f64(w_uv)
    q = f64(q_bt)
    H = q.shape[0]
    n_kv = latent_b.shape[0]
    U = index_set(tok_row, n_kv)
    if U.size == 0:
        return np.zeros((H, uv.shape[1])), np.full(H, -math.inf)
    c = f64(latent_b[U])
    out = np.zeros((H, uv.shape[1]))
    lse = np.zeros(H)
    for h in range(H):
        q_lat = uk[h].T @ q[h]
        o_lat, lse[h] = attend_row(q_lat, c, c, scale)
        out[h] = uv[h] @ o_lat
    return out, lse


def absorb_q(q_rows, w_uk) -> np.ndarray:
    """``q~[n, h, :] = W_UK[h]^T q[n, h, :]`` (``[n, H, d] -> [n, H, L]``)."""
    q = f64(q_rows)
    uk = f64(w_uk)
    return np.einsum("nhd,hdl->nhl", q, uk)


def absorb_out(o_lat_rows, w_uv) -> np.ndarray:
    """``o[n, h, :] = W_UV[h] o~[n, h, :]`` (``[n, H, L] -> [n, H, dv]``)."""
    o = f64(o_lat_rows)
    uv = f64(w_uv)
    return np.einsum("nhl,hdl->nhd", o, uv)


# ---------------------------------------------------------------------------
# S9: indexer query / key preparation (RoPE, Walsh-Hadamard rotation)
# ---------------------------------------------------------------------------
def rope_neox(x, pos: int, n_rope: int, theta: float) -> np.ndarray:
    """NEOX rotary embedding of the first ``n_rope`` values of ``x`` (last axis).

    [ik-2063] PR #2045 "What it does": the rope part of the indexer query and
    key gets NEOX RoPE; the K-shift commit adds that GLM-DSA has no RoPE
    scaling (no extension, attention factor 1, frequency scale 1), so the
    rotation is the plain one and rotations compose.  NEOX pairs value ``i``
    with value ``i + n_rope/2`` (the halves, not neighbours) and turns pair ``i``
    by the angle ``pos * theta**(-2i/n_rope)``.  READING: ``theta`` (the RoPE
    base) is not on the pages; it is an argument.  Values past ``n_rope`` are
    returned unchanged.
    """
    x = f64(x).copy()
    if n_rope % 2:
        raise ValueError("n_rope must be even")
    half = n_rope // 2
    for i in range(half):
        ang = float(pos) * float(theta) ** (-2.0 * i / n_rope)
        c, s = math.cos(ang), math.sin(ang)
        a = x[..., i].copy()
        b = x[..., i + half].copy()
        x[..., i] = a * c - b * s
        x[..., i + half] = b * c + a * s
    return x


def sylvester_hadamard(n: int) -> np.ndarray:
    """The Sylvester Hadamard matrix of order ``n`` (a power of two):
    ``H_1 = [1]``, ``H_2m = [[H_m, H_m], [H_m, -H_m]]`` ([ik-2063] K-shift commit:
    the indexer's Hadamard input is filled with the Sylvester construction)."""
    if n < 1 or n & (n - 1):
        raise ValueError("Hadamard order must be a power of two")
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def hadamard_rotate(x) -> np.ndarray:
    """``H x / sqrt(D)`` along the last axis: the orthonormal Walsh-Hadamard rotation
    ([ik-2063] decode-cache commit: indexer q and k are rotated, which leaves every
    q.k unchanged and helps the precision of the cached keys)."""
    x = f64(x)
    D = x.shape[-1]
    return x @ sylvester_hadamard(D).T / math.sqrt(D)


def index_rotate(x, pos, n_rope: int, theta: float, ln_w=None, ln_b=None, eps: float = 1e-6,
                 layer_norm_first: bool = False, hadamard: bool = True) -> np.ndarray:
    """Prepare indexer queries (``[n, H_I, D]``) or keys (``[n, 1, D]``) for the score.

    [ik-2063] PR #2045 "What it does": indexer_q is split into a rope part and a
    nope part, the rope part gets NEOX RoPE, and the two are concatenated;
    indexer_k is LayerNorm-ed (with bias) and then treated the same way.  The
    decode-cache commit rotates both by the Walsh-Hadamard matrix before the
    key is cached, and the K-shift commit states the cached key as
    ``H * concat(RoPE(k_pe, pos), k_nope)``.  READING: the rope part is the first
    ``n_rope`` values ("split rope(64)/nope(64)", and the rope part comes first
    in the cached concat), so split and concat leave the layout unchanged; the
    rotation is the orthonormal ``H / sqrt(D)``.  ``pos[r]`` is row r's absolute
    position.
    """
    x = f64(x)
    out = np.empty_like(x)
    for r in range(x.shape[0]):
        y = x[r]
        if layer_norm_first:
            y = layer_norm(y, ln_w, ln_b, eps)
        y = rope_neox(y, int(pos[r]), n_rope, theta)
        if hadamard:
            y = hadamard_rotate(y)
        out[r] = y
    return out


# ---------------------------------------------------------------------------
# S2 in FP8: e4m3 indexer operands
# ---------------------------------------------------------------------------
E4M3_MAX = 448.0


def e4m3_grid() -> np.ndarray:
    """The non-negative finite values of the e4m3 format (1 sign, 4 exponent bits
    with bias 7, 3 mantissa bits, no infinities; the all-ones code is NaN),
    ascending: subnormals ``m * 2**-9`` (m = 0..7), then ``2**(e-7) * (1 + m/8)``
    for e = 1..15, m = 0..7, without e = 15, m = 7.  [ik-2063] ships the
    indexer's tensors in F8_E4M3."""
    vals = [m * 2.0 ** -9 for m in range(8)]
    for e in range(1, 16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            vals.append(2.0 ** (e - 7) * (1 + m / 8))
    return np.array(vals)


def e4m3_round(y) -> np.ndarray:
    """Round to the nearest e4m3 value, ties to the even code (even mantissa).

    Inputs beyond the largest value's rounding range (|y| >= 464, halfway to the
    next binade step) raise: the quantiser below scales every vector into range."""
    y = f64(y)
    if np.any(np.abs(y) >= 464.0):
        raise ValueError("value outside the e4m3 range")
    grid = e4m3_grid()
    a = np.abs(y)
    hi = np.clip(np.searchsorted(grid, a, side="left"), 1, grid.size - 1)
    lo = hi - 1
    d_lo, d_hi = a - grid[lo], grid[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))  # codes alternate even/odd along the grid
    q = np.where(pick_hi, grid[hi], grid[lo])
    q = np.where(a == grid[hi], grid[hi], q)
    return np.copysign(q, y)


def fp8_quantize(x):
    """Quantise each vector (last axis) to e4m3 with one fp32 scale.

    READING (the pages name only the F8_E4M3 format): each query-head vector and
    each key row gets ``s = amax / 448``; the codes are ``e4m3(x * (448 / amax))``
    with the reciprocal and the product rounded to fp32, as a kernel computes
    them (the rounding decides the code, so it runs in the kernel's precision).
    A zero vector has scale 1 and zero codes.  Returns (codes, scales) with
    ``x ~= codes * scales[..., None]``.
    """
    x32 = np.asarray(f64(x), dtype=np.float32)
    amax = np.abs(x32).max(axis=-1)
    safe = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
    inv = (np.float32(E4M3_MAX) / safe).astype(np.float32)
    y = (x32 * inv[..., None]).astype(np.float32)
    codes = e4m3_round(y.astype(np.float64))
    scales = np.where(amax > 0, (safe / np.float32(E4M3_MAX)).astype(np.float32), np.float32(1.0))
    return codes, scales.astype(np.float64)


def index_scores_fp8_row(q_row, keys, w_row, scale: float) -> np.ndarray:
    """``I[s] = sum_h w_h * relu(scale * sq_h * sk_s * (q^_h . k^_s))`` with e4m3 codes
    q^, k^ and their scales from :func:`fp8_quantize` ([fak-sparse] §3 score with
    FP8 operands).  The code dot products are exact in float64."""
    qc, qs = fp8_quantize(q_row)          # [H, D], [H]
    kc, ks = fp8_quantize(keys)           # [n, D], [n]
    dots = qc @ kc.T                      # [H, n]
    act = np.maximum(0.0, float(scale) * (qs[:, None] * ks[None, :]) * dots)
    return (f64(w_row)[:, None] * act).sum(axis=0) + 0.0
