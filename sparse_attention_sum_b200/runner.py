"""Convenience layer over the C ABI: allocates outputs and workspaces with torch
and chains the libdsa entry points.  No arithmetic happens here; every step
is one libdsa call.

* :func:`dsa_layer`   -- S1-S5: indexer scores, top-k, sparse MLA attend
  (``dsa_layer_forward``).
* :func:`kpool_layer` -- S6-S8 with S2-S4 over pools: LayerNorm + pooling,
  pool scores, pool top-k (as a set, in pool order), expand_selection, absorbed NoPE MLA attend.
* :func:`dsa_layer_fp8` -- the layer with the FP8 indexer: quantise the queries,
  FP8 scores against a key cache held as e4m3 codes, top-k set, sparse attend.
* :func:`index_share_stack` -- IndexShare over a stack of layers: the layers
  :func:`computes_own_selection` names run the whole layer, the others reuse
  the selection of the last such layer (``idx_in``).
"""
from __future__ import annotations

from typing import Dict, Optional

import torch

from . import (BF16, F32, OP_LAYER_FORWARD, Dims, absorb_out, absorb_q, expand_selection, fp8_quantize,
               index_scores, index_scores_fp8, index_topk_fp8, layer_forward, pool_states, sparse_attend, topk,
               topk_set, workspace_size)


def _code(dtype: torch.dtype) -> int:
    if dtype == torch.float32:
        return F32
    if dtype == torch.bfloat16:
        return BF16
    raise ValueError(f"unsupported dtype {dtype}")


def layer_dims(q_idx, k_idx, q, k, vd: int, top_k: int) -> Dims:
    """Dims of a token-mode layer call from tensor shapes.

    q_idx [B,T,H_I,D_I], k_idx [B,S,D_I], q [B,T,H,kd], k [B,S,Hk,kd] or a
    shared latent [B,S,kd] (Hk = 1).
    """
    B, T, HI, DI = q_idx.shape
    S = k_idx.shape[1]
    H, kd = q.shape[2], q.shape[3]
    Hk = 1 if k.dim() == 3 else k.shape[2]
    return Dims(batch=B, n_q=T, n_kv=S, idx_heads=HI, idx_dim=DI, top_k=top_k, heads=H,
                kv_heads=Hk, kd=kd, vd=vd, kpool=0, out_width=top_k, dtype=_code(q.dtype))


class LayerBuffers:
    """Outputs and workspace of :func:`dsa_layer`, reusable across calls."""

    def __init__(self, dims: Dims, device, out_dtype, with_idx: bool = True, with_lse: bool = False):
        rows = dims.batch * dims.n_q
        self.out = torch.empty(dims.batch, dims.n_q, dims.heads, dims.vd, dtype=out_dtype, device=device)
        self.idx = torch.empty(dims.batch, dims.n_q, dims.top_k, dtype=torch.int32, device=device) \
            if with_idx else None
        self.lse = torch.empty(dims.batch, dims.n_q, dims.heads, dtype=torch.float32, device=device) \
            if with_lse else None
        nbytes = workspace_size(dims, OP_LAYER_FORWARD)
        self.ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)
        self.rows = rows


def dsa_layer(dims: Dims, q_idx, k_idx, w, idx_scale, q_pos, kv_start, kv_len, q, k, v,
              attn_scale, k_row_stride: int, v_row_stride: int, bufs: Optional[LayerBuffers] = None,
              idx_in=None, stream=None) -> LayerBuffers:
    """One call of ``dsa_layer_forward``; returns the buffers holding out/idx/lse."""
    if bufs is None:
        bufs = LayerBuffers(dims, q.device, q.dtype)
    layer_forward(dims, q_idx, k_idx, w, idx_scale, q_pos, kv_start, kv_len, q, k, k_row_stride, v,
                  v_row_stride, attn_scale, bufs.out, lse=bufs.lse, idx_in=idx_in, idx_out=bufs.idx,
                  ws=bufs.ws, stream=stream)
    return bufs


class Fp8Buffers:
    """Per-call FP8 query codes and scales of :func:`dsa_layer_fp8`."""

    def __init__(self, dims: Dims, device):
        shape = (dims.batch, dims.n_q, dims.idx_heads)
        self.q_codes = torch.empty(*shape, dims.idx_dim, dtype=torch.uint8, device=device)
        self.q_scales = torch.empty(*shape, dtype=torch.float32, device=device)


def dsa_layer_fp8(dims: Dims, q_idx, k_codes, k_scales, w, idx_scale, q_pos, kv_start, kv_len, q, k, v,
                  attn_scale, k_row_stride: int, v_row_stride: int, bufs: Optional[LayerBuffers] = None,
                  fp8: Optional[Fp8Buffers] = None, stream=None, k_idx=None) -> LayerBuffers:
    """The layer with the FP8 indexer as libdsa calls: dsa_fp8_quantize of the queries, then
    dsa_index_scores_fp8 against the key cache's e4m3 codes and scales (quantised once, when the keys
    were written) and dsa_topk_set, or dsa_index_topk_fp8 when there is one query per sequence, then
    dsa_sparse_attend.  ``k_idx`` (the bf16 keys) is not read."""
    if bufs is None:
        bufs = LayerBuffers(dims, q.device, q.dtype)
    if fp8 is None:
        fp8 = Fp8Buffers(dims, q.device)
    B, T, S = dims.batch, dims.n_q, dims.n_kv
    scores = bufs.ws[: B * T * S * 4].view(torch.float32).view(B, T, S)
    fp8_quantize(q_idx, fp8.q_codes, fp8.q_scales, stream=stream)
    if dims.n_q == 1:
        # one query per sequence: the fused selection (same keys, no score matrix)
        index_topk_fp8(dims, fp8.q_codes, fp8.q_scales, k_codes, k_scales, w, idx_scale, q_pos, kv_start, kv_len,
                       dims.top_k, bufs.idx, stream=stream)
    else:
        index_scores_fp8(dims, fp8.q_codes, fp8.q_scales, k_codes, k_scales, w, idx_scale, q_pos, kv_start, kv_len,
                         scores, stream=stream)
        topk_set(dims, scores, q_pos, kv_start, kv_len, dims.top_k, bufs.idx, stream=stream)
    sparse_attend(dims, q, k, k_row_stride, v, v_row_stride, bufs.idx, dims.top_k, attn_scale, bufs.out,
                  lse=bufs.lse, stream=stream)
    return bufs


def computes_own_selection(il: int) -> bool:
    """IndexShare schedule (ik_llama.cpp PR #2063, IndexShare commit): layer ``il`` runs its own
    indexer and top-k iff ``il <= 1`` or ``il % 4 == 2``; every other layer reuses the selection of
    the most recent layer that did."""
    return il <= 1 or il % 4 == 2


def index_share_stack(layers, bufs=None, stream=None):
    """Runs ``dsa_layer`` over a stack with IndexShare.

    ``layers`` is a list of ``(dims, kwargs)`` pairs in layer order, ``kwargs`` as for
    :func:`dsa_layer`; every layer's dims must have the same batch, n_q, n_kv and top_k.
    Returns one :class:`LayerBuffers` per layer; a reusing layer's ``idx`` is the shared selection
    tensor itself (the one it attended over).  Layer 0 must compute its own selection."""
    out = []
    shared = None
    for il, (dims, kw) in enumerate(layers):
        b = bufs[il] if bufs is not None else LayerBuffers(dims, kw["q"].device, kw["q"].dtype)
        if computes_own_selection(il):
            dsa_layer(dims, **kw, bufs=b, stream=stream)
            shared = b.idx
        else:
            if shared is None:
                raise ValueError("layer 0 must compute its own selection")
            dsa_layer(dims, **kw, bufs=b, idx_in=shared, stream=stream)
            b.idx = shared
        out.append(b)
    return out


class KpoolBuffers:
    """Intermediates and outputs of :func:`kpool_layer`."""

    def __init__(self, B, T, S, HI, DI, kpool, select_k, out_width, H, dqk, L, dv, device,
                 dtype=torch.bfloat16):
        P = S // kpool
        self.pooled = torch.empty(B, P, DI, dtype=dtype, device=device)
        self.n_pools = torch.empty(B, dtype=torch.int32, device=device)
        self.pool_scores = torch.empty(B, T, P, dtype=torch.float32, device=device)
        self.pool_idx = torch.empty(B, T, select_k, dtype=torch.int32, device=device)
        self.tok_idx = torch.empty(B, T, out_width, dtype=torch.int32, device=device)
        self.q_lat = torch.empty(B, T, H, L, dtype=dtype, device=device)
        self.o_lat = torch.empty(B, T, H, L, dtype=dtype, device=device)
        self.out = torch.empty(B, T, H, dv, dtype=dtype, device=device)


def kpool_dims(B, T, S, HI, DI, kpool, select_k, out_width, H, L, dtype=torch.bfloat16) -> Dict[str, Dims]:
    """Dims of each call of the kpool pipeline."""
    code = _code(dtype)
    P = S // kpool
    return {
        "pool": Dims(batch=B, n_q=T, n_kv=S, idx_heads=HI, idx_dim=DI, top_k=select_k, heads=H,
                     kv_heads=1, kd=L, vd=L, kpool=kpool, out_width=out_width, dtype=code),
        "index": Dims(batch=B, n_q=T, n_kv=P, idx_heads=HI, idx_dim=DI, top_k=select_k, heads=H,
                      kv_heads=1, kd=L, vd=L, kpool=kpool, out_width=out_width, dtype=code),
        "attend": Dims(batch=B, n_q=T, n_kv=S, idx_heads=HI, idx_dim=DI, top_k=out_width, heads=H,
                       kv_heads=1, kd=L, vd=L, kpool=0, out_width=out_width, dtype=code),
    }


def kpool_layer(dims: Dict[str, Dims], q_idx, k_raw, gate, ln_w, ln_b, ln_eps, w, idx_scale, q_pos,
                kv_start, kv_len, q_nope, latent, w_uk, w_uv, attn_scale,
                bufs: KpoolBuffers, stream=None) -> KpoolBuffers:
    """The kpool NoPE DSA layer as a chain of libdsa calls."""
    dp, di, da = dims["pool"], dims["index"], dims["attend"]
    pool_states(dp, k_raw, gate, ln_w, ln_b, ln_eps, kv_start, kv_len, bufs.pooled, bufs.n_pools,
                stream=stream)
    index_scores(di, q_idx, bufs.pooled, w, idx_scale, q_pos, kv_start, kv_len, bufs.pool_scores,
                 stream=stream)
    # the attention reads the expanded tokens as a set, so the pools are selected as one (key order, as the
    # token layer lists its selection); dsa_topk ranks the same pools
    topk_set(di, bufs.pool_scores, q_pos, kv_start, kv_len, di.top_k, bufs.pool_idx, stream=stream)
    expand_selection(dp, bufs.pool_idx, q_pos, kv_start, kv_len, bufs.n_pools, bufs.tok_idx,
                     stream=stream)
    L = da.kd
    absorb_q(da, q_nope, q_nope.shape[-1], w_uk, L, bufs.q_lat, stream=stream)
    sparse_attend(da, bufs.q_lat, latent, L, latent, L, bufs.tok_idx, da.out_width, attn_scale,
                  bufs.o_lat, stream=stream)
    absorb_out(da, bufs.o_lat, L, w_uv, w_uv.shape[1], bufs.out, stream=stream)
    return bufs
