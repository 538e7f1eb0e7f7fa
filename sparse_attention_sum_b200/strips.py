"""Balanced causal strips: one long causal prefill split across ranks by query rows.

The query rows of a causal prefill are independent and the keys are read-only, so rank j can take a
contiguous strip of rows [a_j, b_j) and needs only the keys up to the strip's last query position; its
outputs (attention rows, selections, log-sum-exps) stay on that rank.  A row's cost grows with the keys it
sees, up to top_k, so strips of equal row counts carry very unequal work: :func:`causal_strips` splits the
summed row cost evenly instead.  When the keys arrive sharded (each rank wrote the indexer keys and latent
rows of its own tokens), :func:`gather_key_strips` is the one collective: an all-gather that gives every rank
the whole key prefix.  No kernel reads another GPU's memory.  :func:`run_strip` is one ``dsa_layer_forward``
call on a strip; every step of the layer runs in libdsa.
"""
from __future__ import annotations

from typing import Dict, List, NamedTuple, Optional, Sequence

import numpy as np
import torch

from . import runner

# Cost of a query row, in units of one (query, selected key) pair of the attend, from the measured prefill
# layer (T = S = 4096, top_k = 2048, H = 128, one B200): the attend takes about 0.41 ns per pair over the
# whole GPU, a row boundary of its persistent clusters costs about as much as 200 pairs, and the indexer
# scores a visible key in about 0.053 of the attend's time per pair.
ROW_COST_PAIRS = 200.0
INDEX_COST_RATIO = 0.053


class Strip(NamedTuple):
    """Query rows [a, b) of the sequence and the number of keys they read (key rows [0, key_end))."""
    a: int
    b: int
    key_end: int


def row_costs(q_pos: Sequence[int], top_k: int, kv_start: int = 0) -> np.ndarray:
    """Estimated cost of each query row: min(visible keys, top_k) attended pairs, the indexer's share of
    its visible keys, and a fixed per-row cost; a row that sees no key (a query before kv_start) costs 0."""
    pos = np.asarray(q_pos, dtype=np.float64)
    visible = np.clip(pos - kv_start + 1.0, 0.0, None)
    return np.where(visible > 0, np.minimum(visible, top_k) + INDEX_COST_RATIO * visible + ROW_COST_PAIRS, 0.0)


def causal_strips(q_pos: Sequence[int], world: int, top_k: int, kv_start: int = 0,
                  n_keys: Optional[int] = None) -> List[Strip]:
    """Split the query rows of one sequence (positions ``q_pos``, host integers) into ``world``
    contiguous strips whose summed :func:`row_costs` are as equal as whole rows allow: strip j ends at
    the row boundary nearest to j/world of the total.  ``key_end`` of a strip is one past its largest
    query position (at most ``n_keys``); an empty strip reads no key."""
    if world < 1:
        raise ValueError(f"world must be >= 1 (got {world})")
    pos = np.asarray(q_pos, dtype=np.int64)
    n = int(pos.shape[0])
    cum = np.concatenate([[0.0], np.cumsum(row_costs(pos, top_k, kv_start))])   # cum[i]: rows [0, i)
    total = cum[-1]
    bounds = [0]
    for j in range(1, world):
        target = total * j / world
        i = int(np.searchsorted(cum, target, side="left"))          # first boundary with cum >= target
        if i > 0 and target - cum[i - 1] < cum[min(i, n)] - target:
            i -= 1
        bounds.append(min(n, max(bounds[-1], i)))
    bounds.append(n)
    strips = []
    for j in range(world):
        a, b = bounds[j], bounds[j + 1]
        key_end = int(pos[a:b].max()) + 1 if b > a else 0
        if n_keys is not None:
            key_end = min(key_end, int(n_keys))
        strips.append(Strip(a, b, max(0, key_end)))
    return strips


def run_strip(t: Dict[str, torch.Tensor], strip: Strip, vd: int, top_k: int, idx_scale: float,
              attn_scale: float, bufs: Optional[runner.LayerBuffers] = None, stream=None):
    """``dsa_layer_forward`` on the query rows of ``strip`` of a one-sequence layer held in ``t`` (device
    tensors ``q_idx [1,T,H_I,D_I]``, ``k_idx [1,S,D_I]``, ``w [1,T,H_I]``, ``q_pos [1,T]``, ``kv_start [1]``,
    ``kv_len [1]``, ``q [1,T,H,kd]`` and the shared latent ``latent [1,S,kd]``), against the key rows
    [0, strip.key_end).  Returns the strip's :class:`runner.LayerBuffers` (``out``, ``idx``, ``lse`` hold
    its rows), or None for an empty strip."""
    if t["q"].shape[0] != 1:
        raise ValueError("causal strips split one sequence: batch must be 1")
    a, b, ke = strip
    if b <= a:
        return None
    if ke <= 0:
        raise ValueError("a strip with query rows needs at least one key row")
    q_idx, w, q_pos, q = t["q_idx"][:, a:b], t["w"][:, a:b], t["q_pos"][:, a:b], t["q"][:, a:b]
    k_idx, lat = t["k_idx"][:, :ke], t["latent"][:, :ke]
    kv_len = torch.clamp(t["kv_len"], max=ke)
    kd = lat.shape[-1]
    dims = runner.layer_dims(q_idx, k_idx, q, lat, vd, top_k)
    if bufs is None:
        bufs = runner.LayerBuffers(dims, q.device, q.dtype, with_idx=True, with_lse=True)
    return runner.dsa_layer(dims, q_idx, k_idx, w, idx_scale, q_pos, t["kv_start"], kv_len, q, lat, lat,
                            attn_scale, kd, kd, bufs=bufs, stream=stream)


def gather_key_strips(local: Sequence[torch.Tensor], strips: Sequence[Strip], group=None) -> List[torch.Tensor]:
    """All-gather of key rows written sharded: on rank j each tensor of ``local`` holds the rows
    [strips[j].a, strips[j].b) of one key array (token rows on axis 0, e.g. the indexer keys
    ``[rows, D_I]`` and the latent ``[rows, kd]``).  Returns, on every rank, each array's rows
    [0, strips[-1].b) in token order.  One all-gather per array, of the longest strip's rows (shorter strips
    are padded, and the padding is dropped)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if len(strips) != world:
        raise ValueError(f"{len(strips)} strips for {world} ranks")
    longest = max(s.b - s.a for s in strips)
    out = []
    for x in local:
        padded = torch.zeros((longest,) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
        padded[: x.shape[0]] = x
        parts = [torch.empty_like(padded) for _ in range(world)]
        dist.all_gather(parts, padded, group=group)
        out.append(torch.cat([parts[j][: s.b - s.a] for j, s in enumerate(strips)], dim=0))
    return out
