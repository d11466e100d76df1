"""The benchmark's multi-rank bookkeeping on CPU with two gloo ranks: every
rank runs its own batch (no data-path collective), the job time is the
maximum over ranks and the rate counts all ranks' work."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r "took" 10 + r ms for the timed steps and 20 + 2r for e2e
        ms, e2e = bench.max_over_ranks([10.0 + rank, 20.0 + 2 * rank], torch.device("cpu"), world)
        rate = bench.weak_scaling_rate(1000, world, 5, ms)
        q.put((rank, ms, e2e, rate))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, e2e, rate in res:
        assert ms == 11.0 and e2e == 22.0          # slowest rank on both ranks
        assert rate == pytest.approx(1000 * 2 * 5 / 0.011)


def test_single_rank_is_identity():
    assert bench.max_over_ranks([3.5, 4.0], None, 1) == [3.5, 4.0]
    assert bench.weak_scaling_rate(10, 1, 4, 2.0) == pytest.approx(20000.0)
