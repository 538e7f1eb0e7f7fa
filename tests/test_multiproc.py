"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The DSA path shards into independent problems (one replica of the workload per
GPU, weak scaling), so the only collectives are the plumbing ones bench.py uses:
a barrier around the timed region and an all-reduce(MAX) of the step time.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    import bench
    r, w, local = bench.dist_setup(world)
    assert (r, w, local) == (rank, world, rank)
    assert dist.get_backend() == "gloo"
    bench.barrier(w)
    local_time = 0.25 * (rank + 1)            # each rank's own step-time sum
    slowest = bench.max_over_ranks(local_time, w)
    bench.barrier(w)
    q.put((rank, slowest, bench.replica_seed("prefill", rank)))
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_ranks_take_the_slowest_rank_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [x[1] for x in res] == [0.5, 0.5]          # max over ranks, seen by every rank
    assert res[0][2] != res[1][2]                      # each replica draws its own inputs


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.dist_setup(1) == (0, 1, 0) or os.environ.get("WORLD_SIZE", "1") != "1"
    assert bench.max_over_ranks(1.5, 1) == 1.5
    assert bench.replica_seed("prefill", 0) is None      # rank 0 runs the standard seeded workload
