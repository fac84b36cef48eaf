"""Multi-rank host logic of bench.py on CPU: two gloo ranks (world size 2).

The path shards over sequences with no data-path collective; the only
cross-rank steps are the barrier and the maximum of the per-rank step time.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    w, r, _ = bench.dist_env()
    step_ms = 10.0 + 5.0 * rank                 # rank 1 is the slow one
    slowest = bench.max_over_ranks(step_ms)
    value = bench.aggregate_value(w, 32768, slowest)
    seed = bench.rank_seed(2, r)
    dist.barrier()
    q.put((r, w, slowest, value, seed))
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_step():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, s0, v0, seed0), (r1, w1, s1, v1, seed1) = res
    assert (w0, w1) == (2, 2)
    assert s0 == s1 == 15.0                      # max over ranks
    assert v0 == v1 == pytest.approx(2 * 32768 / 0.015)
    assert seed0 != seed1                        # each rank draws its own sequence


def test_single_process_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.aggregate_value(1, 100, 1000.0) == pytest.approx(100.0)
