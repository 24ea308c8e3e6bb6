"""Host logic of bench.py's multi-process path ("replicas only": every rank runs its own replica;
the job's time is the slowest rank's, its throughput the sum over ranks), run as world_size-2
gloo process groups on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(world)
    ms = [4.0, 6.0][rank]                  # rank 1 is slower
    value, slowest = bench.job_value(10.0, ms, world)
    q.put((rank, value, slowest, bench.max_over_ranks(float(rank + 1), world)))
    dist.destroy_process_group()


def test_job_value_is_sum_over_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, value, slowest, mx in res:
        assert slowest == 6.0                      # the slowest rank's time
        assert abs(value - 2 * 10.0 / 6e-3) < 1e-6  # all ranks' units over that time
        assert mx == 2.0


def test_job_value_single_process():
    import bench
    value, ms = bench.job_value(5.0, 2.0, 1)
    assert ms == 2.0 and abs(value - 2500.0) < 1e-9
