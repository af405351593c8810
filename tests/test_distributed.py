"""Multi-rank plumbing of bench.py on CPU with the gloo backend (world size 2).

The benchmark's data path has no collective: every rank runs its own batch
(weak scaling).  What the ranks share is the timing: the job's step time is
the maximum over ranks, and throughput counts all ranks' tokens.  These
tests run that host logic in two gloo processes; no GPU is involved.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.rank_env()
        assert (r, w, lr) == (rank, world, rank)
        # each rank "measured" a different step time; the slowest one counts
        t = bench.max_over_ranks(10.0 + 5.0 * rank, dist)
        v = bench.job_throughput(w, 32768, t)
        dist.barrier()
        out[rank] = (t, v)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_agree_on_max_time_and_job_throughput():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    port = _free_port()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == out[1]
    t, v = out[0]
    assert t == 15.0
    assert v == pytest.approx(world * 32768 / 0.015)


def test_single_process_defaults():
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.rank_env() == (0, 1, 0)
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(1, 100, 10.0) == pytest.approx(10000.0)
