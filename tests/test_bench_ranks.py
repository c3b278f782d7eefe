"""The benchmark's multi-rank aggregation on CPU with two gloo ranks: every rank
runs its own replica, the reported time is the slowest rank's and the throughput
counts every rank's tokens."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    # rank r measured (1 + r) ms per step and (2 + r) ms end to end
    ms, e2e = bench.slowest_rank(1.0 + rank, 2.0 + rank, world, "cpu")
    q.put((rank, ms, e2e, bench.job_throughput(16, world, ms)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, e2e, value in got:
        assert ms == 2.0 and e2e == 3.0
        assert value == pytest.approx(16 * 2 / 2e-3)


def test_single_rank_is_identity():
    import bench
    assert bench.slowest_rank(1.5, 2.5, 1, "cpu") == (1.5, 2.5)
    assert bench.job_throughput(16, 1, 0.5) == pytest.approx(32000.0)
