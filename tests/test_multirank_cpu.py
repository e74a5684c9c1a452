"""The multi-GPU path is N independent replicas (the work is independent per
request, layer and KV head; nothing is exchanged).  Its host logic -- every
rank takes the same collective steps, the job time is the slowest rank's, the
job throughput counts the bytes of all ranks -- is checked here with two gloo
ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [3.0, 5.0][rank]                      # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, world, "cpu")
        value = bench.job_throughput(326e6, world, ms_max)
        dist.barrier()
        q.put((rank, ms_max, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_sum_the_bytes():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms_max, value in out:
        assert ms_max == 5.0
        assert value == pytest.approx(2 * 326e6 / 5e-3 / 1e9)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(2.5, 1, "cpu") == 2.5
    assert bench.job_throughput(1e9, 1, 1.0) == pytest.approx(1000.0)
