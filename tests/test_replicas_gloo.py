"""The multi-GPU path is replicas only: each rank runs the whole workload and the
ranks share nothing but a barrier and a max-over-ranks of the timings.  That
host logic is exercised here with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r "took" 1.0 + r seconds for 10 steps of 3e12 FLOP each
        secs = bench.reduce_max(1.0 + rank, dist)
        total = bench.reduce_sum(10 * 3e12, dist)
        dist.barrier()
        out[rank] = (secs, total, total / secs / 1e12)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_replica_aggregation():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(90)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(world):
        secs, total, value = res[r]
        assert secs == 2.0            # the slowest rank's time
        assert total == 2 * 10 * 3e12  # work of all replicas
        assert abs(value - 30.0) < 1e-9


def test_single_process_reductions_are_identity():
    import bench

    assert bench.reduce_max(1.5) == 1.5
    assert bench.reduce_sum(7.0) == 7.0
    assert bench.attn_flops(4, 16, 4096, 4096, 128, True) == 274877906944.0
    assert bench.attn_flops(2, 16, 8192, 8192, 128, True, backward=True) == 2.5 * 549755813888.0

