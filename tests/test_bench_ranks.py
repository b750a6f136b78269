"""The multi-rank side of bench.py on CPU: two gloo ranks, each with its own
timings, must both see the per-entry maximum (the slowest rank sets the job
time), and the job throughput counts the work of every rank (weak scaling:
independent replicas, no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r: total 10 + r ms, components r-dependent, one rank slower per entry
        mine = torch.tensor([10.0 + rank, 1.0 + 2 * rank, 5.0 - rank, 0.5, 3.0 * (rank + 1), 7.0], dtype=torch.float64)
        got = bench.max_over_ranks(mine.clone(), world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_of_each_timing():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = [11.0, 3.0, 5.0, 0.5, 6.0, 7.0]
    assert res[0] == want and res[1] == want


def test_single_rank_needs_no_process_group():
    t = torch.tensor([1.0, 2.0], dtype=torch.float64)
    assert bench.max_over_ranks(t, 1) == [1.0, 2.0]


@pytest.mark.parametrize("world", [1, 2, 8])
def test_job_throughput_counts_every_rank(world):
    # 2 TFLOP per rank in 1 ms on each of `world` ranks
    assert bench.job_tflops(world, 2e12, 1.0) == pytest.approx(2000.0 * world)
