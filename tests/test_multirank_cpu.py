"""The replicas path of bench.py on two CPU ranks (gloo): the slowest rank's time sets the
whole-job rate, and every rank takes the same collective steps."""
import os
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_seconds = [0.010, 0.025][rank]
    slowest = bench.max_over_ranks(local_seconds, world, dist, "cpu")
    rate = bench.whole_job_rate(16384, 10, world, slowest)
    dist.barrier()
    out[rank] = (slowest, rate)
    dist.destroy_process_group()


def test_two_rank_rate_uses_the_slowest_rank():
    port = 29500 + os.getpid() % 1000
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == res[1]
    slowest, rate = res[0]
    assert slowest == pytest.approx(0.025)
    assert rate == pytest.approx(2 * 16384 * 10 / 0.025)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.5, 1) == 0.5
    assert bench.whole_job_rate(100, 4, 1, 2.0) == 200.0
