"""Replica aggregation of the benchmark with two gloo ranks on the CPU: the
whole-job value is every rank's tokens over the slowest rank's time."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = [10.0, 25.0][rank]
    tokens = [4096, 4096][rank]
    value, ms_max, total = bench.replica_throughput(ms, tokens, dist)
    q.put((rank, value, ms_max, total))
    dist.barrier()
    dist.destroy_process_group()


def test_two_replicas_take_max_time_and_sum_tokens():
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
    for rank, value, ms_max, total in res:
        assert ms_max == 25.0 and total == 8192
        assert value == pytest.approx(8192 / 0.025)


def test_single_process_needs_no_group():
    import bench
    value, ms, total = bench.replica_throughput(20.0, 4096)
    assert (ms, total) == (20.0, 4096) and value == pytest.approx(4096 / 0.02)
