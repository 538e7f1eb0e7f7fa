"""Balanced causal strips (one long prefill split by query rows across ranks): the strip plan and the
all-gather of sharded key rows, on the CPU (gloo, world size 2)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("T,world,top_k,kv_start", [(4096, 2, 2048, 0), (4096, 8, 2048, 0), (1000, 3, 96, 0),
                                                     (5000, 4, 2048, 700), (131072, 8, 2048, 0), (7, 3, 4, 0)])
def test_strips_cover_the_rows_and_balance_their_cost(T, world, top_k, kv_start):
    from sparse_attention_sum_b200 import strips as S
    pos = np.arange(T)
    plan = S.causal_strips(pos, world, top_k, kv_start=kv_start)
    assert len(plan) == world
    assert plan[0].a == 0 and plan[-1].b == T
    for s0, s1 in zip(plan, plan[1:]):
        assert s0.b == s1.a                                         # contiguous, in order
    for s in plan:
        assert s.a <= s.b
        assert s.key_end == (int(pos[s.a:s.b].max()) + 1 if s.b > s.a else 0)
    cost = S.row_costs(pos, top_k, kv_start)
    # each boundary sits at the row boundary nearest its target, so a strip exceeds its share by at most
    # one row's cost
    share = cost.sum() / world
    for s in plan:
        assert cost[s.a:s.b].sum() <= share + cost.max() + 1e-6
    # strips of causal rows: later rows see more keys, so equal-cost strips get shorter
    if world > 1 and T >= 1000 and kv_start == 0:
        lengths = [s.b - s.a for s in plan]
        assert lengths[0] > lengths[-1]


def test_row_cost_follows_the_visible_keys():
    from sparse_attention_sum_b200 import strips as S
    top_k = 16
    pos = np.arange(40)
    c = S.row_costs(pos, top_k, kv_start=10)
    assert np.all(c[:10] == 0)                                       # queries before the first key
    vis = pos[10:] - 10 + 1
    expect = np.minimum(vis, top_k) + S.INDEX_COST_RATIO * vis + S.ROW_COST_PAIRS
    assert np.allclose(c[10:], expect)
    assert np.all(np.diff(c[10:]) > 0)                               # more visible keys, more cost


def test_one_rank_takes_every_row_and_key_end_is_capped():
    from sparse_attention_sum_b200 import strips as S
    plan = S.causal_strips(np.arange(300) + 50, 1, 64, n_keys=320)
    assert plan == [S.Strip(0, 300, 320)]
    with pytest.raises(ValueError):
        S.causal_strips(np.arange(10), 0, 4)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gather_worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from sparse_attention_sum_b200 import strips as S
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    T = 1003
    plan = S.causal_strips(np.arange(T), world, 256)
    g = torch.Generator().manual_seed(3)
    k_idx = torch.randn(T, 128, generator=g).to(torch.bfloat16)      # every rank draws the same arrays
    latent = torch.randn(T, 576, generator=g).to(torch.bfloat16)
    mine = plan[rank]
    full = S.gather_key_strips([k_idx[mine.a:mine.b].clone(), latent[mine.a:mine.b].clone()], plan)
    q.put((rank, torch.equal(full[0], k_idx), torch.equal(full[1], latent), [tuple(s) for s in plan]))
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_sharded_key_rows_gather_to_the_whole_prefix():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_gather_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert all(r[1] and r[2] for r in res)
    plan = res[0][3]
    assert plan == res[1][3] and plan[0][1] - plan[0][0] != plan[1][1] - plan[1][0]   # uneven strips
