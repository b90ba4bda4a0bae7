"""The N > 1 bench path runs independent replicas (one per GPU, no data
exchange): its only collective steps are the barriers and the max-over-ranks
reduction of the timed region.  Checked here with two gloo ranks on CPU."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as tdist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 30.0][rank]  # rank 1 is the slow replica
        tdist.barrier()
        ms = bench.max_over_ranks(local_ms, world, "cpu")
        tflops = bench.job_tflops(1e12, ms, steps=10, world=world)
        tdist.barrier()
        results[rank] = (ms, tflops)
    finally:
        tdist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank_time():
    world = 2
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert results[0] == results[1]
    ms, tflops = results[0]
    assert ms == 30.0
    # 2 ranks x 10 launches x 1 TFLOP in 30 ms
    assert tflops == pytest.approx(2 * 10 * 1.0 / 0.030)


def test_single_rank_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.0, 1, "cpu") == 7.0
    assert bench.job_tflops(2e12, 20.0, steps=5, world=1) == pytest.approx(500.0)
