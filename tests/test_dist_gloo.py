"""Host logic of the multi-GPU benchmark (replicas, weak scaling) on CPU with gloo.

Two ranks with different per-rank times: the reported time must be the max over
ranks and the throughput the whole job's; the reference arm runs on rank 0 only.
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
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench

    t_local = 1.0 + rank          # rank 1 is slower
    t = bench.reduce_over_ranks(t_local, dist, "cpu", "max")
    tmin = bench.reduce_over_ranks(t_local, dist, "cpu", "min")
    v = bench.job_throughput(per_rank_units=8, steps=10, world=world, max_seconds=t)
    dist.barrier()
    q.put((rank, t, tmin, v))
    dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_throughput():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, tmin, v in res:
        assert t == 2.0 and tmin == 1.0
        assert v == 2 * 8 * 10 / 2.0


def test_reference_arm_other_ranks_do_no_work():
    import bench

    class A:
        warmup, steps, gpus, workload = 3, 1, 2, "tiny_m64"

    assert bench.run_reference(A(), bench.workloads.CONFIGS["tiny"], 64, rank=1, world=2) is None
