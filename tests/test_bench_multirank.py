"""The multi-rank path of bench.py on CPU: two gloo ranks (replicas, no data-path
collective) reduce their timings to the slowest rank's, and the whole-job throughput
counts every rank's tokens against that time."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    import torch.distributed as td
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    td.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r "measured" 10 + r ms in total, 5 - r ms for another quantity
        got = bench.reduce_max_over_ranks([10.0 + rank, 5.0 - rank], td, "cpu")
        q.put((rank, got))
    finally:
        td.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    results = dict(q.get(timeout=10) for _ in range(world))
    for r in range(world):
        assert results[r] == [11.0, 5.0]


def test_whole_job_value_counts_every_rank():
    # 16384 tokens per rank, 2 ranks, 10 steps in 5 ms (max over ranks): 0.5 ms per step
    assert bench.whole_job_tokens_per_s(16384, 2, 5.0, 10) == pytest.approx(2 * 16384 / 0.5e-3)
