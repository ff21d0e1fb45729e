"""The multi-GPU form of the bench is N independent replicas: no collective
in the data path, the job's time is the slowest rank's and its throughput
sums every rank's tokens. Two gloo ranks on the CPU check that arithmetic
and that every rank reaches the same collective steps."""

from __future__ import annotations

import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms = [100.0, 250.0][rank]  # rank 1 is the slow one
        value, ms_max = bench.job_throughput(256, world, ms)
        out.put((rank, value, ms_max))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank_and_sum_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, ms_max in res:
        assert ms_max == 250.0
        assert abs(value - 2 * 256 / 0.25) < 1e-9
