"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, each with its
own (different) local time; every rank must see the slowest time and the
whole-job rate must count both ranks' work over it."""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local_s = [0.5, 2.0][rank]
    rate, slow = bench.whole_job_rate(dist, world, 1000.0, local_s, torch.device("cpu"))
    m = bench.max_over_ranks(dist, float(rank + 7), torch.device("cpu"))
    out[rank] = (rate, slow, m)
    dist.barrier()
    dist.destroy_process_group()


def test_whole_job_rate_uses_the_slowest_rank():
    port = 29500 + (os.getpid() % 2000)
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank, args=(2, port, out), nprocs=2, join=True)
    for r in range(2):
        rate, slow, m = out[r]
        assert slow == 2.0
        assert rate == pytest.approx(2 * 1000.0 / 2.0)
        assert m == 8.0


def test_single_process_passes_through():
    sys.path.insert(0, ROOT)
    import bench
    rate, slow = bench.whole_job_rate(None, 1, 10.0, 0.5, torch.device("cpu"))
    assert (rate, slow) == (20.0, 0.5)
