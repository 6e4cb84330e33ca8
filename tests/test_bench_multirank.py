"""The N>1 bench plumbing on CPU: two gloo ranks, max-over-ranks timing and
whole-job throughput (every rank runs an independent replica; no collective
touches the data path)."""
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


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env() == (rank, world, rank)
        # rank r reports a step time of 10 + 5r ms and an e2e time of 30 - r ms
        got = bench.reduce_max([10.0 + 5 * rank, 30.0 - rank])
        q.put((rank, got, bench.job_tflops(world, 2e12, got[0])))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_two_ranks_take_the_max_and_scale_weakly(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, tf in res:
        assert got == [10.0 + 5 * (world - 1), 30.0]
        # 2 ranks x 2 TFLOP per step in 15 ms
        assert abs(tf - world * 2.0 / 0.015) < 1e-9


def test_single_rank_reduce_is_identity():
    import bench
    assert bench.reduce_max([1.5, 2.5]) == [1.5, 2.5]
    assert abs(bench.job_tflops(1, 1e12, 1000.0) - 1.0) < 1e-12
