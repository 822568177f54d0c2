"""The replica (weak-scaling) plumbing of bench.py with two gloo ranks on CPU: every rank runs its
own units, the job's time is the slowest rank's (all-reduce MAX), and the whole-job throughput is
units x ranks / that time.  No data-path collective exists: each rank's key switches are local."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from datetime import timedelta
    import torch.distributed as dist
    import bench
    r, w, lr = bench.rank_env()
    dist.init_process_group("gloo", rank=r, world_size=w, timeout=timedelta(seconds=300))
    ms = 100.0 + 50.0 * rank                     # rank 1 is the slow one
    ms_max = bench.max_over_ranks(ms, w)
    value = bench.job_throughput(16, w, ms_max)
    dist.barrier()
    dist.destroy_process_group()
    q.put((r, w, lr, ms_max, value))


@pytest.mark.parametrize("world", [2])
def test_replica_timing_two_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(600)             # a fresh process's first torch import can take a minute or more
        assert p.exitcode == 0
    res = sorted(q.get(timeout=60) for _ in range(world))
    for r, (rank, w, lr, ms_max, value) in enumerate(res):
        assert (rank, w, lr) == (r, world, r)
        assert ms_max == 150.0                               # max over ranks
        assert abs(value - 16 * world / 0.150) < 1e-6        # units x ranks / slowest time


def test_single_process_defaults(monkeypatch):
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.rank_env() == (0, 1, 0)
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.job_throughput(10, 1, 1000.0) == 10.0
