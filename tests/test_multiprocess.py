"""Multi-rank logic of bench.py on CPU: two gloo ranks, each with its own
problem of the same shape, timed as the max over ranks (no GPU)."""

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
    import bench
    from head_weighted_relu_b200 import workloads as W
    wl = W.WORKLOADS["tiny_int_512"]
    mine = bench.rank_workload(wl, rank)
    inp = W.generate(mine, "cpu")
    elapsed = 10.0 + rank          # each rank's own time
    t = bench.max_over_ranks(elapsed, world, device="cpu")
    dist.barrier()
    out[rank] = (mine.seed, float(inp["q"].float().sum()), t)
    dist.destroy_process_group()


def test_two_gloo_ranks_have_independent_problems_and_max_time():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    (s0, q0, t0), (s1, q1, t1) = res[0], res[1]
    assert s0 != s1 and q0 != q1                 # different problems
    assert t0 == t1 == 11.0                      # every rank sees the slowest
