"""GPU parity of the indexer query / key preparation step (dsa_index_rotate) against the CPU oracle.

Small cases compare every value; the full-size cases run in the launch configuration bench.py times
(prefill: 4096 tokens x 64 query heads and 4096 keys; decode: 64 new keys written into a 64 x 32768
key cache) and compare sampled rows value by value, plus the rows that must stay untouched.

Tolerance, from the arithmetic: the angles are exact to double precision and every other step runs
in fp32 (about 1e-6 of the row's largest value after the LayerNorm and seven butterfly stages), then
the store rounds once.  A value may therefore differ from the f64 oracle by one unit in the last
place of the output type (2^-7 relative for bf16, 2^-23 for fp32) plus 1e-5 of the largest magnitude
in its head vector.
"""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
import sparse_attention_sum_b200 as dsa
import workloads

pytestmark = pytest.mark.gpu

THETA = 10000.0
EPS = 1e-6


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dsa.lib()  # fail loudly if the library is missing
    yield
    assert dsa.get_device_status() == 0


def _oracle(inp, rows, n_rope, ln, had):
    x = inp["x"][rows]
    pos = O.i64(inp["pos"][rows])
    return O.index_rotate(x, pos, n_rope, THETA, inp["ln_w"] if ln else None, inp["ln_b"] if ln else None, EPS,
                          layer_norm_first=ln, hadamard=had)


def _assert_close(got, ref, out_dtype):
    got = got.detach().to(torch.float64).cpu().numpy()
    rel = 2.0 ** -7 if out_dtype == torch.bfloat16 else 2.0 ** -23
    bound = rel * np.abs(ref) + 1e-5 * np.abs(ref).max(axis=-1, keepdims=True)
    err = np.abs(got - ref) - bound
    assert not (err > 0).any(), f"{int((err > 0).sum())} values outside the bound (worst excess {err.max():.3g})"


def _rotate(inp, out, n_rope, ln, had, out_rows=None, x=None):
    d = {k: v.cuda() for k, v in inp.items()}
    dsa.index_rotate(d["x"] if x is None else x, out, n_rope, THETA, pos=d["pos"], layer_norm=ln, ln_w=d["ln_w"],
                     ln_b=d["ln_b"], ln_eps=EPS, hadamard=had,
                     out_rows=None if out_rows is None else out_rows.cuda())
    torch.cuda.synchronize()


CASES = [
    # name, n_rows, heads, dim, in dtype, out dtype, n_rope, layer_norm, hadamard
    ("queries bf16", 257, 64, 128, "bf16", torch.bfloat16, 64, False, True),
    ("keys bf16", 70, 1, 128, "bf16", torch.bfloat16, 64, True, True),
    ("dim 32 f32", 45, 3, 32, "f32", torch.float32, 32, True, True),
    ("dim 64 no rope", 33, 9, 64, "bf16", torch.float32, 0, True, True),
    ("dim 64 rope only", 20, 17, 64, "f32", torch.bfloat16, 64, False, False),
    ("dim 128 n_rope 8", 70, 1, 128, "bf16", torch.bfloat16, 8, True, False),
    ("dim 128 all rope", 19, 12, 128, "f32", torch.float32, 128, True, True),
    # rows of whole 32-head blocks take the four-lanes-per-vector kernel: every n_rope it serves
    ("32 heads all rope f32", 33, 32, 128, "f32", torch.float32, 128, True, True),
    ("64 heads no rope", 21, 64, 128, "bf16", torch.bfloat16, 0, False, True),
    ("96 heads rope only", 9, 96, 128, "bf16", torch.float32, 64, True, False),
]


@pytest.mark.parametrize("name,n_rows,heads,dim,in_dt,out_dt,n_rope,ln,had", CASES, ids=[c[0] for c in CASES])
def test_small_cases_every_value(name, n_rows, heads, dim, in_dt, out_dt, n_rope, ln, had):
    inp = workloads.rotate_inputs(n_rows, heads, dim, seed=21, dtype=in_dt, mean=0.5 if ln else 0.0,
                                  std=2.0 if ln else 1.0)
    inp["pos"][0] = 0          # position 0: RoPE is the identity
    inp["pos"][-1] = 32767     # the largest angle of the decode workload
    out = torch.empty(n_rows, heads, dim, dtype=out_dt, device="cuda")
    _rotate(inp, out, n_rope, ln, had)
    _assert_close(out, _oracle(inp, slice(None), n_rope, ln, had), out_dt)


def test_strided_rows_in_and_out():
    """Rows wider than heads*dim on both sides (a fused projection output, a padded cache)."""
    n_rows, heads, dim = 50, 4, 128
    inp = workloads.rotate_inputs(n_rows, heads, dim, seed=22)
    wide = torch.zeros(n_rows, heads * dim + 64, dtype=torch.bfloat16)
    wide[:, 32:32 + heads * dim] = inp["x"].reshape(n_rows, -1)
    xin = wide.cuda()[:, 32:32 + heads * dim].unflatten(1, (heads, dim))
    big = torch.full((n_rows, heads * dim + 256), 7.0, dtype=torch.bfloat16, device="cuda")
    out = big[:, 128:128 + heads * dim].unflatten(1, (heads, dim))
    _rotate(inp, out, 64, False, True, x=xin)
    _assert_close(out, _oracle(inp, slice(None), 64, False, True), torch.bfloat16)
    assert (big[:, :128] == 7.0).all() and (big[:, 128 + heads * dim:] == 7.0).all()


def test_rows_aligned_to_eight_bytes_only():
    """A row stride of 132 values (4-value aligned, not 8): the dim-128 kernel's 16-byte accesses
    cannot serve it, so the general kernel runs; both layouts give the oracle's values."""
    n_rows, heads, dim = 37, 1, 128
    inp = workloads.rotate_inputs(n_rows, heads, dim, seed=29, mean=0.5, std=2.0)
    wide = torch.zeros(n_rows, 132, dtype=torch.bfloat16)
    wide[:, 4:132] = inp["x"].reshape(n_rows, -1)
    xin = wide.cuda()[:, 4:132].unflatten(1, (heads, dim))
    out = torch.empty(n_rows, heads, dim, dtype=torch.bfloat16, device="cuda")
    _rotate(inp, out, 64, True, True, x=xin)
    assert dsa.last_kernels() == ["index_rotate"]
    _assert_close(out, _oracle(inp, slice(None), 64, True, True), torch.bfloat16)


def test_in_place():
    inp = workloads.rotate_inputs(40, 8, 128, seed=23)
    x = inp["x"].cuda().clone()
    _rotate(inp, x, 64, True, True, x=x)
    _assert_close(x, _oracle(inp, slice(None), 64, True, True), torch.bfloat16)


def test_keys_go_to_their_cache_slots_and_nothing_else_changes():
    """Keys scattered into a cache by slot; slot -1 and slots past the capacity are not written."""
    n_rows, cap = 300, 512
    inp = workloads.rotate_inputs(n_rows, 1, 128, seed=24, mean=0.5, std=2.0)
    g = torch.Generator().manual_seed(24)
    slots = torch.randperm(cap, generator=g)[:n_rows].to(torch.int32)
    slots[[3, 77, 150, 299]] = -1
    slots[[10, 200]] = cap + torch.tensor([0, 1000], dtype=torch.int32)
    cache = torch.full((cap, 1, 128), -3.0, dtype=torch.bfloat16, device="cuda")
    _rotate(inp, cache, 64, True, True, out_rows=slots)
    ok = ((slots >= 0) & (slots < cap)).nonzero().flatten()
    ref = _oracle(inp, ok, 64, True, True)
    _assert_close(cache[slots[ok].long().cuda()], ref, torch.bfloat16)
    untouched = torch.ones(cap, dtype=torch.bool)
    untouched[slots[ok].long()] = False
    assert (cache[untouched.cuda()] == -3.0).all()


def test_no_rows_and_all_slots_skipped():
    inp = workloads.rotate_inputs(8, 2, 64, seed=25)
    cache = torch.full((8, 2, 64), 5.0, dtype=torch.float32, device="cuda")
    empty = workloads.rotate_inputs(0, 2, 64, seed=25)
    _rotate(empty, cache, 64, False, True)
    _rotate(inp, cache, 64, False, True, out_rows=torch.full((8,), -1, dtype=torch.int32))
    assert (cache == 5.0).all()


def test_rotated_queries_and_keys_give_the_same_scores_on_the_gpu():
    """The Hadamard rotation leaves the indexer scores unchanged (ik_llama.cpp #2045): rotate q and k
    with and without it, then score both on the GPU."""
    T, HI, D = 96, 8, 128
    qi = workloads.rotate_inputs(T, HI, D, seed=26, dtype="f32")
    ki = workloads.rotate_inputs(T, 1, D, seed=27, dtype="f32", mean=0.5, std=2.0)
    ki["pos"] = qi["pos"] = torch.arange(T, dtype=torch.int32)
    g = torch.Generator().manual_seed(28)
    w = (torch.randn(1, T, HI, generator=g) / 8).cuda()
    dims = dsa.Dims(batch=1, n_q=T, n_kv=T, idx_heads=HI, idx_dim=D, top_k=16, heads=1, kv_heads=1, kd=D, vd=D,
                    kpool=0, out_width=16, dtype=dsa.F32)
    pos = torch.arange(T, dtype=torch.int32, device="cuda")
    start = torch.zeros(1, dtype=torch.int32, device="cuda")
    length = torch.full((1,), T, dtype=torch.int32, device="cuda")
    scores = []
    for had in (True, False):
        q = torch.empty(T, HI, D, dtype=torch.float32, device="cuda")
        k = torch.empty(T, 1, D, dtype=torch.float32, device="cuda")
        _rotate(qi, q, 64, False, had)
        _rotate(ki, k, 64, True, had)
        s = torch.empty(1, T, T, dtype=torch.float32, device="cuda")
        dsa.index_scores(dims, q.unsqueeze(0), k.view(1, T, D), w, 0.1, pos, start, length, s)
        torch.cuda.synchronize()
        scores.append(s.cpu().double().numpy())
    vis = np.isfinite(scores[1])
    assert np.array_equal(vis, np.isfinite(scores[0])) and vis.sum() == T * (T + 1) // 2
    scale = np.abs(scores[1][vis]).max()
    assert np.abs(scores[0][vis] - scores[1][vis]).max() <= 1e-5 * scale


# ------------------------------------------------------------ full size
def _sample(n, k, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, n - 1], rng.choice(n, k, replace=False)]))


def test_full_size_prefill_queries_and_keys_sampled_rows():
    """Prefill: 4096 tokens x 64 query heads, and 4096 keys with the LayerNorm."""
    q_in = workloads.rotate_inputs(4096, 64, 128, seed=1, pos_max=4096)
    q_in["pos"] = torch.arange(4096, dtype=torch.int32)
    k_in = workloads.rotate_inputs(4096, 1, 128, seed=2, mean=0.5, std=2.0)
    k_in["pos"] = torch.arange(4096, dtype=torch.int32)
    q_out = torch.empty(4096, 64, 128, dtype=torch.bfloat16, device="cuda")
    k_out = torch.empty(4096, 1, 128, dtype=torch.bfloat16, device="cuda")
    _rotate(q_in, q_out, 64, False, True)
    _rotate(k_in, k_out, 64, True, True)
    rows = _sample(4096, 14, 3)
    _assert_close(q_out[torch.from_numpy(rows).cuda()], _oracle(q_in, rows, 64, False, True), torch.bfloat16)
    _assert_close(k_out, _oracle(k_in, slice(None), 64, True, True), torch.bfloat16)


def test_full_size_decode_keys_into_the_cache():
    """Decode: each of 64 sequences appends its new key at position 32767 of a 32768-row cache."""
    B, S = 64, 32768
    k_in = workloads.rotate_inputs(B, 1, 128, seed=4, mean=0.5, std=2.0)
    k_in["pos"] = torch.full((B,), S - 1, dtype=torch.int32)
    slots = (torch.arange(B, dtype=torch.int32) * S + (S - 1))
    cache = torch.zeros(B * S, 1, 128, dtype=torch.bfloat16, device="cuda")
    _rotate(k_in, cache, 64, True, True, out_rows=slots)
    _assert_close(cache[slots.long().cuda()], _oracle(k_in, slice(None), 64, True, True), torch.bfloat16)
    assert int((cache != 0).any(dim=2).sum()) <= B
    assert not cache[(slots - 1).long().cuda()].any()
