"""The N>1 path's host logic on CPU: two gloo ranks join, time a fake step, take the max
over ranks and form the whole-job throughput, as bench.py does over NCCL."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from exact_io_aware_64_b200 import dist as fa_dist


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    info = fa_dist.rank_info()
    fa_dist.init(info, "gloo", timeout_s=60)
    fa_dist.barrier(info)
    my_time = 1.0 + rank          # rank 1 is the slow one
    t = fa_dist.max_over_ranks(my_time, info)
    value = fa_dist.aggregate_throughput(10.0, t, info)
    seed = fa_dist.replica_seed(5, info)
    fa_dist.barrier(info)
    fa_dist.shutdown(info)
    out.put((rank, t, value, seed))


def test_two_gloo_ranks_take_the_max_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in results] == [2.0, 2.0]           # everyone sees the slowest rank
    assert all(abs(r[2] - 2 * 10.0 / 2.0) < 1e-12 for r in results)
    assert results[0][3] != results[1][3]                  # disjoint inputs per replica


def test_single_rank_is_a_noop():
    info = fa_dist.RankInfo(0, 1, 0)
    fa_dist.init(info, "gloo")
    fa_dist.barrier(info)
    assert fa_dist.max_over_ranks(3.5, info) == 3.5
    assert fa_dist.aggregate_throughput(8.0, 2.0, info) == 4.0
    fa_dist.shutdown(info)
