"""The bench's multi-rank host logic on two gloo ranks (CPU): the step time is
the maximum over ranks of each rank's device time, and the whole-job value
counts every rank's batch (weak scaling, no data-path exchange)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r measured (10 + r) ms for the step loop and (30 - r) ms end to end
        got = bench.max_over_ranks([10.0 + rank, 30.0 - rank], world, "cpu")
        dist.barrier()
        out[rank] = tuple(got)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        # every rank sees the same maxima: 11 ms (rank 1's loop), 30 ms (rank 0's e2e)
        assert out[0] == out[1] == (11.0, 30.0)


def test_single_rank_is_identity_and_job_value_counts_all_ranks():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.0], 1) == [3.0, 4.0]
    tokens, value = bench.job_throughput(4, 8, 2.0)
    assert tokens == 32 and value == pytest.approx(32 / 2e-3)
