"""The N > 1 plumbing of bench.py on CPU with gloo ranks (world size 2).

The SPTS path does not shard inside a sequence, so several GPUs run
independent replicas; the only cross-rank steps are the barrier around the
timed region and the max-over-ranks of its duration.  Those run here on CPU.
"""

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
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = 10.0 + 5.0 * rank                         # rank 1 is the slow one
        mx = bench.max_over_ranks(ms, torch.device("cpu"))
        q.put((rank, mx, bench.job_throughput(32768, world, mx)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[1] for g in got] == [15.0, 15.0]
    assert all(abs(g[2] - 32768 * 2 / 0.015) < 1e-6 for g in got)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.job_throughput(100, 1, 1000.0) == 100.0
