"""The benchmark's multi-GPU path on CPU: world_size 2 over gloo.  Each rank
runs its own replica (no data-path collective); the job time is the max over
ranks and the throughput counts every rank's work."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    per_rank_ms = [40.0, 55.0][rank]
    got = bench.reduce_max(per_rank_ms, world)
    tflops = bench.job_tflops(6.5e12, 10, world, got)
    q.put((rank, got, tflops))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, tflops in res:
        assert got == 55.0                                  # max over ranks
        assert abs(tflops - 2 * 6.5e12 * 10 / 0.055 / 1e12) < 1e-9
    import bench
    assert bench.reduce_max(7.0, 1) == 7.0                  # single rank: identity
