"""The multi-GPU bench path on the host: two gloo ranks on the CPU take the
slowest rank's time (max over ranks) and report weak-scaling job throughput.
The GPU runs use the same functions over NCCL."""
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


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [1.5, 2.25][rank]  # ms per step seen by this rank
        worst = bench.max_over_ranks(mine, True)
        dist.barrier()
        q.put((rank, worst, bench.job_throughput(world, 1.0e12, worst, "TFLOP/s")))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, worst, value in got:
        assert worst == pytest.approx(2.25)
        # 2 ranks x 1 TFLOP of work in the slowest rank's 2.25 ms
        assert value == pytest.approx(2 * 1.0e12 / 2.25e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.0, False) == 3.0
    assert bench.job_throughput(1, 2.0e9, 1.0, "GB/s") == pytest.approx(2000.0)
