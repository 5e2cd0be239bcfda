"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): each
rank runs its own replica of the workload and the job's step time is the
slowest rank's."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, l = bench.dist_env()
        assert (w, r, l) == (world, rank, rank)
        # rank 1 is the slow one: 30 ms over 10 steps vs 20 ms
        local_ms = 20.0 + 10.0 * rank
        value, step_ms = bench.job_throughput(tokens_per_rank=16, world=world, local_ms_total=local_ms, steps=10)
        bench.barrier()
        wl = bench.rank_workload("small_mla_bf16", rank)
        q.put((rank, value, step_ms, wl.seed))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_and_max_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, value, step_ms, seed in res:
        assert step_ms == pytest.approx(3.0)                   # the slowest rank's 30 ms / 10 steps
        assert value == pytest.approx(2 * 16 / 3.0e-3)        # both ranks' tokens over that time
    assert res[0][3] != res[1][3]                              # each rank draws its own sequences


def test_single_process_reduce_is_identity():
    assert bench.reduce_max(1.5) == 1.5
    assert bench.job_throughput(16, 1, 10.0, 10) == (16 / 1e-3, 1.0)
