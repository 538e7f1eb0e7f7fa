"""Seeded synthetic inputs: shapes, determinism and structure (no GPU)."""
import torch

import workloads


def test_tiny_is_deterministic_and_integer():
    a = workloads.make("tiny")
    b = workloads.make("tiny")
    for key in a.tensors:
        assert torch.equal(a[key], b[key]), key
    assert a["q_idx"].abs().max() <= 4 and torch.equal(a["q_idx"], a["q_idx"].round())
    assert set(a["w"].unique().tolist()) <= {0.5, 1.0, 2.0, 4.0}
    assert a["q"].dtype == torch.float32 and a.kv_heads == a.heads


def test_small_prefill_shapes_and_dtypes():
    wl = workloads.make("prefill", T=256)
    assert wl["q_idx"].shape == (1, 256, 64, 128) and wl["q_idx"].dtype == torch.bfloat16
    assert wl["k_idx"].shape == (1, 256, 128)
    assert wl["latent"].shape == (1, 256, 576)
    assert wl["q"].shape == (1, 256, 128, 576)
    assert wl["w"].dtype == torch.float32
    assert wl["q_pos"].tolist() == [list(range(256))]
    # latent ~ N(0, 0.5^2)
    assert 0.45 < wl["latent"].float().std().item() < 0.55


def test_chunked_hot_spots_are_disjoint_runs():
    g = torch.Generator().manual_seed(3)
    starts = workloads.hot_spot_runs(g, 32768, 51, 64)
    assert len(starts) == 51 and len(set(starts.tolist())) == 51
    s = sorted(starts.tolist())
    assert all(b - a >= 64 for a, b in zip(s, s[1:]))
    wl = workloads.make("chunked", T=64, S=4096)
    assert wl["q_pos"][0, 0].item() == 4096 - 64
    # hot keys sit ~3 above the rest on every channel
    m = wl["k_idx"][0].float().mean(dim=1)
    assert (m > 1.5).sum().item() == (4096 // 10) // 64 * 64


def test_kpool_padding_and_widths():
    wl = workloads.make("kpool", T=64, pads=(0, 3, 17, 20))
    assert wl["kv_start"].tolist() == [0, 3, 17, 20]
    assert wl.out_width == 512 * 4 + 3
    assert wl["w_uk"].shape == (64, 128, 512)
