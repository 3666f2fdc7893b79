"""The multi-GPU split of one problem, on CPU (no GPU): query rows are
independent problems, so the split is by rows -- contiguous, query-block
aligned ranges of about equal visible-pair count (indexer_partition_rows) --
with the keys replicated on every rank and nothing exchanged.  Two gloo ranks
each compute their part with the oracle from the same sub-problem bench.py
builds; the gathered rows must equal the single-rank result."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASES = {
    "token": dict(S=300, T=300, H=4, D=64, K=16),
    "compressed": dict(S=301, T=75, H=4, D=64, K=8, visibility=1, ratio=4),
    "pooled_offset": dict(S=200, T=330, H=8, D=128, K=16, visibility=2, ratio=4, q_pos0=130),
}


def _workload(name):
    from head_weighted_relu_b200 import workloads as W
    return W.Workload(name, seed=5, values="int", **CASES[name])


def _oracle_rows(wl, inp, r0, r1):
    import oracle
    from head_weighted_relu_b200 import workloads as W
    sub = wl.scaled(S=r1 - r0, q_pos0=wl.q_pos0 + r0)
    bits = lambda t: None if t is None else W.to_host_bits(t)  # noqa: E731
    idx, ln, _, _ = oracle.topk_rows(sub.problem(), bits(inp["q"][r0:r1]), bits(inp["k"]),
                                     bits(inp["w"][r0:r1]), np.arange(r1 - r0),
                                     pool_coef=bits(inp["pool_coef"]))
    return idx, ln


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from head_weighted_relu_b200 import workloads as W
    res = {}
    for name in CASES:
        wl = _workload(name)
        gen_wl, r0, r1 = bench.rank_part(wl, rank, world, "strong")
        inp = W.generate(gen_wl, "cpu")            # every rank draws the same inputs: keys replicated
        idx, ln = _oracle_rows(gen_wl, inp, r0, r1)
        parts = [None] * world
        dist.all_gather_object(parts, (r0, r1, idx, ln))
        res[name] = parts
    t = bench.max_over_ranks(10.0 + rank, world, device="cpu")
    dist.barrier()
    out[rank] = (res, t)
    dist.destroy_process_group()


def test_two_gloo_ranks_split_one_problem_by_rows():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][1] == res[1][1] == 11.0            # every rank sees the slowest time
    from head_weighted_relu_b200 import workloads as W
    for name in CASES:
        wl = _workload(name)
        parts = res[0][0][name]
        assert parts[0][0] == 0 and parts[0][1] == parts[1][0] and parts[1][1] == wl.S
        idx = np.concatenate([p[2] for p in parts])
        ln = np.concatenate([p[3] for p in parts])
        ref_idx, ref_len = _oracle_rows(wl, W.generate(wl, "cpu"), 0, wl.S)
        assert np.array_equal(ln, ref_len), name
        assert np.array_equal(idx, ref_idx), name


@pytest.mark.parametrize("vis,ratio,q_pos0", [(0, 1, 0), (1, 4, 0), (2, 4, 0), (0, 1, 5000), (2, 4, 777)])
def test_partition_rows_cover_and_balance(vis, ratio, q_pos0):
    import bench
    from head_weighted_relu_b200 import indexer as I
    from head_weighted_relu_b200 import workloads as W
    for S, H in ((1, 64), (37, 64), (4099, 64), (20000, 32), (65536, 64)):
        T = S + q_pos0 if vis != 1 else (S + q_pos0) // ratio + 1
        wl = W.Workload("p", S=S, T=T, H=H, D=128, K=2048, visibility=vis, ratio=ratio, q_pos0=q_pos0)
        prob = bench.problem_of(wl)
        qb = min(256 // H, 32)
        per_row = bench.visible_per_row(wl)
        blocks = [per_row[b:b + qb].sum() for b in range(0, S, qb)]
        for n in (1, 2, 3, 4, 8):
            b = I.indexer_partition_rows(prob, n)
            assert len(b) == n + 1 and b[0] == 0 and b[-1] == S
            assert all(x <= y for x, y in zip(b, b[1:]))                      # every row exactly once
            assert all(x % qb == 0 or x == S for x in b)                       # whole query blocks
            share = per_row.sum() / n
            for i in range(n):
                part = per_row[b[i]:b[i + 1]].sum()
                assert abs(part - share) <= max(blocks), (S, n, i, part, share)


def test_partition_rows_rejects_bad_arguments():
    from head_weighted_relu_b200 import indexer as I
    prob = I.make_problem(100, 100, 64, 128, 16)
    for n in (0, -1, 5000):
        with pytest.raises(I.IndexerError) as e:
            I.indexer_partition_rows(prob, n)
        assert e.value.status == 1
