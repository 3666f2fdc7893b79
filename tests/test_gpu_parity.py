"""CUDA path vs the CPU oracle on inputs small enough for the oracle to check
every row, spanning several key tiles, several query blocks and ragged tails."""

import numpy as np
import pytest
import torch

import oracle
from head_weighted_relu_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


def _all_rows(wl):
    return np.arange(wl.S, dtype=np.int64)


def test_tiny_integer_bit_exact(cuda_ok):
    """Integer inputs (every score exact in FP32 and FP64): indices, lengths and
    scores bit-exact on all 512 rows, ties broken by the lower key index."""
    wl = W.WORKLOADS["tiny_int_512"]
    inp = W.generate(wl, "cuda")
    gpu = parity.run_gpu(wl, inp)
    rows = _all_rows(wl)
    parity.assert_exact(gpu, parity.oracle_rows(wl, inp, rows), rows)


@pytest.mark.parametrize("S,T,H,D,K", [
    (1000, 1000, 64, 128, 256),     # token, ragged tile and block tails
    (777, 777, 32, 128, 100),
    (600, 600, 16, 64, 64),
    (300, 300, 8, 128, 40),
    (520, 520, 4, 64, 33),
])
def test_token_gaussian(cuda_ok, S, T, H, D, K):
    wl = W.Workload("t", S=S, T=T, H=H, D=D, K=K, seed=100 + H)
    inp = W.generate(wl, "cuda")
    gpu = parity.run_gpu(wl, inp)
    rows = _all_rows(wl)
    parity.assert_tolerant(wl, gpu, parity.oracle_rows(wl, inp, rows), rows)


def test_integer_many_ties_multi_flush(cuda_ok):
    """Integer scores with K small against long rows: the candidate buffer is cut
    many times, and ties at the threshold must resolve to the lowest indices."""
    wl = W.Workload("ties", S=256, T=3000, H=4, D=64, K=40, q_pos0=3000 - 256, seed=7, values="int")
    inp = W.generate(wl, "cuda")
    gpu = parity.run_gpu(wl, inp)
    rows = _all_rows(wl)
    parity.assert_exact(gpu, parity.oracle_rows(wl, inp, rows), rows)


def test_compressed_m4(cuda_ok):
    wl = W.Workload("csa", S=3001, T=750, H=64, D=128, K=128, visibility=W.COMPRESSED,
                    ratio=4, seed=11)
    inp = W.generate(wl, "cuda")
    gpu = parity.run_gpu(wl, inp)
    rows = _all_rows(wl)
    parity.assert_tolerant(wl, gpu, parity.oracle_rows(wl, inp, rows), rows)


def test_pooled_with_tail(cuda_ok):
    wl = W.Workload("pool", S=1234, T=1234, H=32, D=128, K=256, visibility=W.POOLED,
                    ratio=4, seed=12)
    inp = W.generate(wl, "cuda")
    gpu = parity.run_gpu(wl, inp)
    rows = _all_rows(wl)
    parity.assert_tolerant(wl, gpu, parity.oracle_rows(wl, inp, rows), rows)


def test_pooled_keys_bit_exact(cuda_ok):
    from head_weighted_relu_b200 import indexer as I
    wl = W.Workload("pool", S=64, T=4096, H=32, D=128, K=64, visibility=W.POOLED, ratio=4,
                    seed=13)
    inp = W.generate(wl, "cuda")
    kp = I.pool_keys(inp["k"], inp["pool_coef"], 4)
    torch.cuda.synchronize()
    ref = oracle.pooled_keys(W.to_host_bits(inp["k"]), W.to_host_bits(inp["pool_coef"]), 4)
    assert np.array_equal(W.to_host_bits(kp), ref)


def test_fp8_long_rows(cuda_ok):
    wl = W.Workload("fp8", S=300, T=5000, H=64, D=128, K=512, dtype="fp8", q_pos0=4700, seed=14)
    inp = W.generate(wl, "cuda")
    gpu = parity.run_gpu(wl, inp)
    rows = _all_rows(wl)
    parity.assert_tolerant(wl, gpu, parity.oracle_rows(wl, inp, rows), rows)


def test_kpool_watch_lengths(cuda_ok):
    """Sequences of the lengths 3, 4, 5, 7, 8, 9 ("Module 06 — DSA & KPool",
    §3): each query sees only complete pools, plus its own incomplete tail."""
    from head_weighted_relu_b200 import indexer as I
    for L in (3, 4, 5, 7, 8, 9):
        wl = W.Workload("watch", S=L, T=L, H=32, D=128, K=8, visibility=W.POOLED, ratio=4, seed=L)
        inp = W.generate(wl, "cuda")
        gpu = parity.run_gpu(wl, inp)
        rows = _all_rows(wl)
        ref = parity.oracle_rows(wl, inp, rows)
        gi, gl = gpu[0].cpu().numpy(), gpu[1].cpu().numpy()
        assert np.array_equal(gl, ref["len"]), (L, gl, ref["len"])
        assert np.array_equal(gi, ref["idx"]), (L, gi, ref["idx"])
        assert gi.shape[1] == I.indexer_out_width(I.make_problem(L, L, 32, 128, 8, W.POOLED, 4))


def test_edge_cases(cuda_ok):
    # single query, single key; budget above the history; zero weights (all ties)
    cases = [
        W.Workload("one", S=1, T=1, H=64, D=128, K=4, seed=1),
        W.Workload("k1", S=200, T=200, H=64, D=128, K=1, seed=2),
        W.Workload("kbig", S=130, T=130, H=64, D=128, K=4096, seed=3),
        W.Workload("csa_empty", S=9, T=4, H=64, D=128, K=2, visibility=W.COMPRESSED, ratio=4, seed=4),
    ]
    for wl in cases:
        inp = W.generate(wl, "cuda")
        gpu = parity.run_gpu(wl, inp)
        rows = _all_rows(wl)
        parity.assert_tolerant(wl, gpu, parity.oracle_rows(wl, inp, rows), rows)
    wl = W.Workload("zero_w", S=300, T=300, H=64, D=128, K=50, seed=5)
    inp = W.generate(wl, "cuda")
    inp["w"].zero_()
    gi, gl, gs = parity.run_gpu(wl, inp)
    gi, gl = gi.cpu().numpy(), gl.cpu().numpy()
    for t in range(wl.S):
        n = min(wl.K, t + 1)
        assert gl[t] == n and gi[t, :n].tolist() == list(range(n))


def test_deterministic_and_pair_overlap(cuda_ok):
    from head_weighted_relu_b200 import indexer as I
    wl = W.Workload("det", S=1000, T=1000, H=64, D=128, K=200, seed=21)
    inp = W.generate(wl, "cuda")
    a = parity.run_gpu(wl, inp)
    b = parity.run_gpu(wl, inp)
    for x, y in zip(a, b):
        assert torch.equal(x.nan_to_num(-7.0) if x.is_floating_point() else x,
                           y.nan_to_num(-7.0) if y.is_floating_point() else y)
    shared = I.pair_overlap(a[0], a[1])
    torch.cuda.synchronize()
    # rows 0..K-1 see their whole prefix: shared = length of the even row (the
    # oracle comparison of the pair steps is in test_gpu_pairs.py)
    assert shared[: wl.K // 2].cpu().tolist() == [2 * p + 1 for p in range(wl.K // 2)]


def test_device_status_clean(cuda_ok):
    from head_weighted_relu_b200 import indexer as I
    wl = W.Workload("st", S=500, T=500, H=64, D=128, K=64, seed=31)
    inp = W.generate(wl, "cuda")
    prob = I.make_problem(wl.S, wl.T, wl.H, wl.D, wl.K)
    bufs = I.allocate(prob, "cuda")
    I.topk(inp["q"], inp["k"], inp["w"], wl.K, buffers=bufs)
    assert I.indexer_read_status(bufs[3]) == 0
