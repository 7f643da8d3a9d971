"""The multi-rank path of bench.py on CPU: two gloo ranks agree on the max-over-ranks timings and
on the whole-job (weak-scaling) throughput, as the NCCL ranks do on GPUs."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        elapsed, kernel = 100.0 + 7.0 * rank, 50.0 - rank
        got = bench.max_over_ranks([elapsed, kernel], dist, "cpu")
        value = bench.weak_scaling_value(6.0e11, world, 10, got[0])
        out[rank] = torch.tensor([got[0], got[1], value], dtype=torch.float64)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    world = 2
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    r0, r1 = out[0].tolist(), out[1].tolist()
    assert r0 == r1
    assert r0[0] == 107.0 and r0[1] == 50.0
    assert r0[2] == pytest.approx(2 * 6.0e11 * 10 / 0.107)


def test_single_process_is_a_no_op():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert bench.weak_scaling_value(10.0, 1, 2, 1000.0) == 20.0
