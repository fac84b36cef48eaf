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


# ---------------------------------------------------------------------------
# One prefill split over ranks (bench.py --split-sequence): zig-zag query
# blocks, a position-sharded key cache gathered by one all-gather per tensor.

def test_zigzag_blocks_cover_every_row_once_with_equal_causal_work():
    from sparse_attention_08_b200 import sharding as S
    L = 4096
    for world in (1, 2, 4, 8):
        rows, work = [], []
        for r in range(world):
            blocks = S.zigzag_blocks(L, world, r)
            rows += [i for q0, q1 in blocks for i in range(q0, q1)]
            work.append(sum(sum(p + 1 for p in range(q0, q1)) for q0, q1 in blocks))
        assert sorted(rows) == list(range(L))
        assert max(work) - min(work) <= (L // (2 * world)) ** 2   # equal up to rounding of halves
    with pytest.raises(ValueError):
        S.zigzag_blocks(100, 3, 0)


def test_blocks_as_chunks_reproduce_the_whole_prefill():
    """A block [q0, q1) run as one chunk (len_q = q1 - q0 against the first q1
    keys) sees its rows at positions q0.. : the oracle over the blocks equals
    the oracle over the whole sequence, bit for bit."""
    import numpy as np
    import oracle
    from sparse_attention_08_b200 import sharding as S
    from sparse_attention_08_b200 import workloads as W
    from tests import dsa_cases as C
    wl = W.make_small(H_I=4, d_I=64, H=16, L=96, k=16, integer=True, seed=13)
    args = (C.np_(wl.q8), C.np_(wl.q_scale), C.np_(wl.w), C.np_(wl.k8), C.np_(wl.k_scale),
            C.bits(wl.q), C.bits(wl.kv))
    idx_all, out_all, lse_all = oracle.forward(*args, wl.k, wl.scale)
    world = 3
    seen = np.zeros(96, dtype=bool)
    for r in range(world):
        for q0, q1 in S.zigzag_blocks(96, world, r):
            a = S.block_args(q0, q1)
            qr, kr = a["q_rows"], a["key_rows"]
            assert a["cu_q"] == [0, q1 - q0] and a["cu_k"] == [0, q1]
            idx_b, out_b, lse_b = oracle.forward(args[0][qr], args[1][qr], args[2][qr],
                                                 args[3][kr], args[4][kr], args[5][qr],
                                                 args[6][kr], wl.k, wl.scale)
            assert np.array_equal(idx_b, idx_all[qr])
            assert np.array_equal(out_b, out_all[qr])
            assert np.array_equal(lse_b, lse_all[qr])
            seen[qr] = True
    assert seen.all()


def _gather_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from sparse_attention_08_b200 import sharding as S
    L = 64
    full_f = torch.arange(L * 3, dtype=torch.float32).reshape(L, 3)
    full_b = (torch.arange(L * 5) % 251).to(torch.uint8).reshape(L, 5)
    k0, k1 = S.key_shard(L, world, rank)
    got_f = S.all_gather_rows(full_f[k0:k1])
    got_b = S.all_gather_rows(full_b[k0:k1])
    q.put((rank, bool(torch.equal(got_f, full_f)), bool(torch.equal(got_b, full_b))))
    dist.destroy_process_group()


def test_all_gather_rows_rebuilds_the_sharded_cache_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, True, True), (1, True, True)]
