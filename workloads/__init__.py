"""Seeded synthetic inputs for the DSA layer workloads.

This module only draws random numbers and lays them out; it holds none of the
layer's arithmetic.  Both the CPU oracle (``oracle/``) and the CUDA path read
the tensors it returns, so the two always see identical values.

Every tensor is drawn on the CPU from a ``torch.Generator`` seeded with the
workload's seed, in fp32, and rounded once (round-to-nearest-even) to bf16 for
the bf16 workloads.  Draw order is fixed, so a workload is reproducible on any
machine.

Workload shapes follow the DSA pages:

* the lightning indexer uses one shared 128-wide key head per token and 64
  query heads, top_k 2048 (ik_llama.cpp PR #2063, commit message of #2045:
  "single key head, MQA", "indexer_head_size=128", rope 64 / nope 64);
* the MLA attention reads a shared 576-wide latent row (512 kv_lora + 64 rope)
  whose first 512 columns are the value (the key width differs from the value
  width: fak note "GLM-5.2: the DSA sparse attention moves onto the pure fak
  kernel", section "What changed");
* the kpool NoPE variant pools the indexer keys four at a time from the first
  valid token (metrale ``glm5next_dsa_ref`` module page, invariants list).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch

INVALID = -1

__all__ = ["Workload", "make", "NAMES", "INVALID", "hot_spot_runs", "rotate_inputs"]

NAMES = ("tiny", "prefill", "decode", "chunked", "kpool")


@dataclasses.dataclass
class Workload:
    """One synthetic DSA layer problem (all tensors on the CPU)."""

    name: str
    seed: int
    dtype: str                  # "f32" or "bf16"
    batch: int
    n_q: int
    n_kv: int
    idx_heads: int
    idx_dim: int
    top_k: int
    heads: int
    kv_heads: int
    kd: int
    vd: int
    idx_scale: float
    attn_scale: float
    kpool: int = 0
    select_k: int = 0
    out_width: int = 0
    ln_eps: float = 0.0
    tensors: Dict[str, torch.Tensor] = dataclasses.field(default_factory=dict)

    def __getitem__(self, key: str) -> torch.Tensor:
        return self.tensors[key]

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


def _randn(g: torch.Generator, shape, std: float = 1.0) -> torch.Tensor:
    t = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def _randn_bf16(g: torch.Generator, shape, std: float = 1.0, chunk_rows: int = 4096) -> torch.Tensor:
    """Draw N(0, std^2) in fp32 and round to bf16, chunked along dim 0 to bound memory."""
    out = torch.empty(*shape, dtype=torch.bfloat16)
    flat = out.view(shape[0], -1)
    for r0 in range(0, shape[0], chunk_rows):
        r1 = min(shape[0], r0 + chunk_rows)
        flat[r0:r1] = _randn(g, (r1 - r0, flat.shape[1]), std).to(torch.bfloat16)
    return out


def hot_spot_runs(g: torch.Generator, n_kv: int, n_runs: int, run_len: int) -> torch.Tensor:
    """Start offsets of ``n_runs`` non-overlapping runs of ``run_len`` consecutive keys.

    The key range is cut into ``n_kv // run_len`` aligned slots and ``n_runs``
    distinct slots are drawn without replacement, so runs never overlap.
    """
    slots = n_kv // run_len
    perm = torch.randperm(slots, generator=g)[:n_runs]
    return torch.sort(perm).values * run_len


def _tiny(seed: int) -> Workload:
    g = torch.Generator().manual_seed(seed)
    B, T, HI, DI, H, KD, VD = 1, 64, 4, 32, 8, 32, 24
    wl = Workload("tiny", seed, "f32", B, T, T, HI, DI, 16, H, H, KD, VD,
                  idx_scale=1.0 / 8.0, attn_scale=1.0 / math.sqrt(32.0))
    ts = wl.tensors
    # Integer indexer inputs and power-of-two weights make every score exact.
    ts["q_idx"] = torch.randint(-4, 5, (B, T, HI, DI), generator=g).to(torch.float32)
    ts["k_idx"] = torch.randint(-4, 5, (B, T, DI), generator=g).to(torch.float32)
    wsel = torch.randint(0, 4, (B, T, HI), generator=g)
    ts["w"] = torch.tensor([0.5, 1.0, 2.0, 4.0])[wsel]
    ts["q"] = _randn(g, (B, T, H, KD))
    ts["k"] = _randn(g, (B, T, H, KD))
    ts["v"] = _randn(g, (B, T, H, VD))
    ts["q_pos"] = torch.arange(T, dtype=torch.int32).view(1, T).repeat(B, 1)
    ts["kv_start"] = torch.zeros(B, dtype=torch.int32)
    ts["kv_len"] = torch.full((B,), T, dtype=torch.int32)
    return wl


def _int_vectors(g: torch.Generator, shape, fp8: bool) -> torch.Tensor:
    """Integer indexer vectors: uniform in [-4, 4]; with ``fp8``, uniform in [-7, 7] with one entry
    of every vector (last axis) set to 7, so that every vector's largest magnitude is exactly 7."""
    if not fp8:
        return torch.randint(-4, 5, shape, generator=g)
    x = torch.randint(-7, 8, shape, generator=g)
    pos = torch.randint(0, shape[-1], shape[:-1], generator=g)
    x.scatter_(-1, pos.unsqueeze(-1), 7)
    return x


def _mla_common(name, seed, B, T, S, q_pos, latent_std, hot_spots=False, exact_index=False) -> Workload:
    """The bf16 MLA workloads.  ``exact_index`` swaps the indexer inputs for the
    integer recipe of the tiny workload (q_I, k_I integers in [-4, 4], w in
    {1/2, 1, 2, 4}, indexer scale 1/8) at the same shapes: every score is then a
    multiple of 1/16 below 2^17, exact in fp32 whatever the summation order.
    ``exact_index="fp8"`` draws q_I, k_I in [-7, 7] with each vector's largest
    magnitude exactly 7 (no hot spots): scores stay multiples of 1/16 below 2^19,
    and a per-vector e4m3 quantisation with scale amax/448 is then exact (scale
    1/64, codes 64*x)."""
    g = torch.Generator().manual_seed(seed)
    HI, DI, H, KD, VD = 64, 128, 128, 576, 512
    wl = Workload(name, seed, "bf16", B, T, S, HI, DI, 2048, H, 1, KD, VD,
                  idx_scale=1.0 / 8.0 if exact_index else 1.0 / math.sqrt(128.0),
                  attn_scale=1.0 / math.sqrt(192.0))
    ts = wl.tensors
    if exact_index:
        ts["q_idx"] = _int_vectors(g, (B, T, HI, DI), exact_index == "fp8").to(torch.bfloat16)
    else:
        ts["q_idx"] = _randn_bf16(g, (B, T, HI, DI))
    if exact_index == "fp8" and hot_spots:
        raise ValueError("exact_index='fp8' needs every key's largest magnitude to stay 7 (no hot spots)")
    k_idx = torch.empty(B, S, DI, dtype=torch.bfloat16)
    for b in range(B):
        kb = _int_vectors(g, (S, DI), exact_index == "fp8").to(torch.float32) if exact_index else _randn(g, (S, DI))
        if hot_spots:
            # 10% of the keys (51 runs of 64) get +3 on every indexer-key channel.
            starts = hot_spot_runs(g, S, max(1, (S // 10) // 64), 64)
            for s0 in starts.tolist():
                kb[s0:s0 + 64] += 3.0
        k_idx[b] = kb.to(torch.bfloat16)
    ts["k_idx"] = k_idx
    if exact_index:
        ts["w"] = torch.tensor([0.5, 1.0, 2.0, 4.0])[torch.randint(0, 4, (B, T, HI), generator=g)]
    else:
        ts["w"] = _randn(g, (B, T, HI), std=1.0 / 8.0)
    ts["q"] = _randn_bf16(g, (B * T, H, KD)).view(B, T, H, KD)
    ts["latent"] = _randn_bf16(g, (B * S, KD), std=latent_std).view(B, S, KD)
    ts["q_pos"] = q_pos.to(torch.int32)
    ts["kv_start"] = torch.zeros(B, dtype=torch.int32)
    ts["kv_len"] = torch.full((B,), S, dtype=torch.int32)
    return wl


def _prefill(seed: int, T: int = 4096, exact_index: bool = False) -> Workload:
    q_pos = torch.arange(T).view(1, T)
    return _mla_common("prefill", seed, 1, T, T, q_pos, latent_std=0.5, exact_index=exact_index)


def _decode(seed: int, B: int = 64, S: int = 32768, exact_index: bool = False) -> Workload:
    q_pos = torch.full((B, 1), S - 1)
    return _mla_common("decode", seed, B, 1, S, q_pos, latent_std=0.5, exact_index=exact_index)


def _chunked(seed: int, T: int = 4096, S: int = 32768, exact_index: bool = False) -> Workload:
    q_pos = (S - T + torch.arange(T)).view(1, T)
    return _mla_common("chunked", seed, 1, T, S, q_pos, latent_std=1.0, hot_spots=True,
                       exact_index=exact_index)


def _kpool(seed: int, T: int = 8192, pads=(0, 17, 513, 1029)) -> Workload:
    g = torch.Generator().manual_seed(seed)
    B = len(pads)
    HI, DI, H, DQK, LORA = 32, 128, 64, 128, 512
    KPOOL, SELK = 4, 512
    wl = Workload("kpool", seed, "bf16", B, T, T, HI, DI, SELK, H, 1, LORA, LORA,
                  idx_scale=1.0 / math.sqrt(128.0), attn_scale=1.0 / math.sqrt(128.0),
                  kpool=KPOOL, select_k=SELK, out_width=SELK * KPOOL + KPOOL - 1, ln_eps=1e-6)
    ts = wl.tensors
    ts["q_idx"] = _randn_bf16(g, (B * T, HI, DI)).view(B, T, HI, DI)
    ts["k_raw"] = _randn_bf16(g, (B * T, DI)).view(B, T, DI)
    ts["gate"] = _randn_bf16(g, (B * T, DI)).view(B, T, DI)
    ts["ln_w"] = 1.0 + _randn(g, (DI,), std=0.1)
    ts["ln_b"] = _randn(g, (DI,), std=0.1)
    ts["w"] = _randn(g, (B, T, HI), std=1.0 / 8.0)
    ts["q_nope"] = _randn_bf16(g, (B * T, H, DQK)).view(B, T, H, DQK)
    ts["latent"] = _randn_bf16(g, (B * T, LORA)).view(B, T, LORA)
    ts["w_uk"] = _randn_bf16(g, (H, DQK, LORA), std=1.0 / math.sqrt(LORA))
    ts["w_uv"] = _randn_bf16(g, (H, DQK, LORA), std=1.0 / math.sqrt(LORA))
    ts["q_pos"] = torch.arange(T, dtype=torch.int32).view(1, T).repeat(B, 1)
    ts["kv_start"] = torch.tensor(pads, dtype=torch.int32)
    ts["kv_len"] = torch.full((B,), T, dtype=torch.int32)
    return wl


_BUILDERS = {"tiny": _tiny, "prefill": _prefill, "decode": _decode,
             "chunked": _chunked, "kpool": _kpool}
_DEFAULT_SEEDS = {"tiny": 0, "prefill": 1, "decode": 2, "chunked": 3, "kpool": 4}


def make(name: str, seed: Optional[int] = None, **sizes) -> Workload:
    """Build workload ``name`` (one of :data:`NAMES`).

    ``sizes`` overrides the sequence/batch sizes (``T``, ``S``, ``B``, ``pads``)
    for scaled-down parity cases; the distributions stay the same.  The bf16 MLA
    workloads also take ``exact_index=True`` (integer indexer inputs, see
    ``_mla_common``).
    """
    if name not in _BUILDERS:
        raise KeyError(f"unknown workload {name!r}; expected one of {NAMES}")
    s = _DEFAULT_SEEDS[name] if seed is None else seed
    return _BUILDERS[name](s, **sizes)


def rotate_inputs(n_rows: int, heads: int, dim: int = 128, seed: int = 5, pos_max: int = 32768,
                  dtype: str = "bf16", mean: float = 0.0, std: float = 1.0) -> Dict[str, torch.Tensor]:
    """Inputs of the indexer query / key preparation step (all on the CPU).

    ``x [n_rows, heads, dim]`` ~ N(mean, std^2) (the indexer projections' output;
    queries use 64 heads, keys one), ``pos [n_rows]`` int32 uniform in
    ``[0, pos_max)``, and the key LayerNorm's ``ln_w = 1 + 0.1 N``,
    ``ln_b = 0.1 N`` (fp32), drawn in that order.
    """
    g = torch.Generator().manual_seed(seed)
    x = _randn(g, (n_rows, heads, dim), std)
    if mean:
        x.add_(mean)
    if dtype == "bf16":
        x = x.to(torch.bfloat16)
    pos = torch.randint(0, pos_max, (n_rows,), generator=g, dtype=torch.int32)
    ln_w = 1 + 0.1 * _randn(g, (dim,))
    ln_b = 0.1 * _randn(g, (dim,))
    return {"x": x, "pos": pos, "ln_w": ln_w, "ln_b": ln_b}
