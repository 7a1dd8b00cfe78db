"""The multi-GPU path of bench.py on CPU: two gloo ranks check the
max-over-ranks timing reduction and the whole-job throughput (each rank
verifies its own sequences; no data-path collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 5.0 - rank]           # rank 1 is slower on the first, faster on the second
        got = bench.reduce_max(mine, world)
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_two_rank_max_reduction():
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == [11.0, 5.0]


def test_job_throughput_is_weak_scaling():
    one = bench.job_throughput(1, 64, 100, 10.0)
    four = bench.job_throughput(4, 64, 100, 10.0)
    assert four == pytest.approx(4 * one)
    assert one == pytest.approx(64 * 100 / 0.01)
