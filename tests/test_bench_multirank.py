"""bench.py's multi-process timing path on CPU: two gloo ranks, each with its
own replica time; the job's time is the slowest rank's and the throughput
counts every rank's replica (the path shards into independent replicas, so
there is no data-path collective to test)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    ms = bench.max_over_ranks(1.0 + rank, dist, "cpu")  # rank 1 is the slower one
    out[rank] = (ms, bench.whole_job_gbs(world, 1_000_000, 10, ms))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_whole_job_value():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        for r in range(2):
            ms, gbs = out[r]
            assert ms == 2.0
            assert gbs == pytest.approx(2 * 1_000_000 * 10 / 2e-3 / 1e9)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
