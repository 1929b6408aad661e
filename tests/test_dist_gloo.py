"""The multi-GPU host logic of bench.py on CPU with gloo, world size 2: each
replica draws its own tokens from its own seed, the job time is the max over
ranks, and the job value counts every rank's tokens. (On GPUs the same code
runs over NCCL; the layer itself has no cross-GPU exchange.)"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from workloads import make_x, small_case
        sh = small_case("dist", T=8, d=128, E=4, k=2, F=128, act="swiglu").shape
        x = make_x(sh.with_(seed=bench.replica_seed(sh, rank)))
        t_ms = 10.0 + 5.0 * rank  # a per-rank time; rank 1 is the slowest
        tmax = bench.reduce_max(t_ms, world)
        digest = float(x.float().sum())
        gathered = [None] * world
        dist.all_gather_object(gathered, digest)
        out[rank] = (tmax, bench.job_value(sh.T, 3, world, tmax), gathered)
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    for r in range(world):
        tmax, value, digests = res[r]
        assert tmax == 15.0                       # the slowest rank's time
        assert abs(value - 2 * 8 * 3 / 0.015) < 1e-6
        assert digests[0] != digests[1]           # replicas draw different tokens
