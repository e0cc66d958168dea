"""The N > 1 host path of bench.py on CPU: two gloo ranks, each a replica.

The attention path has no exchange step, so the only cross-rank logic is the
barrier and the max over ranks of the device times; this checks both with a
world of two processes (spawned, 127.0.0.1 rendezvous).
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        per_rank_ms = [120.0, 150.0][rank]
        dist.barrier()
        slowest = bench.reduce_max(per_rank_ms, world, "cpu")
        value = bench.whole_job_tflops(world, 1.5e13, 10, slowest)
        out.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_rank():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, value in res:
        assert slowest == 150.0
        assert value == pytest.approx(2 * 1.5e13 * 10 / 0.150 / 1e12)


def test_single_rank_is_identity():
    import bench

    assert bench.reduce_max(3.5, 1, "cpu") == 3.5
    assert bench.whole_job_tflops(1, 1e12, 1, 1000.0) == pytest.approx(1.0)
