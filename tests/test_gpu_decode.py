"""Decode-like shapes -- a few query rows against a long key range -- where the
indexer cuts each query block's key tiles into ranges spread over the SMs and
merges the per-range top-K lists.  Every row is checked against the oracle,
including ties that straddle range boundaries, every visibility mode, FP8
keys, and the pruning stage (which must leave the result bit-identical)."""

import numpy as np
import pytest
import torch

from head_weighted_relu_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


def _splits(wl) -> int:
    """The key-range split count the library plans for this shape (mirrors the
    host rule), so that each test asserts it exercises the split path."""
    qb = min(256 // wl.H, 32)
    nb = -(-wl.S // qb)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if nb * 2 > sms:
        return 1
    g = wl.q_pos0 + wl.S - 1
    n_keys = wl.T // wl.ratio if wl.visibility == W.POOLED else wl.T
    nvis = g + 1 if wl.visibility == W.TOKEN else (g + 1) // wl.ratio
    nvis = min(nvis, n_keys)
    s = min(sms // nb, (nvis + 127) // 128 // 16, 512)
    return s if s >= 2 else 1


def _rows(wl):
    return np.arange(wl.S, dtype=np.int64)


def test_decode_integer_bit_exact(cuda_ok):
    """Integer inputs with many equal scores: indices, lengths and scores
    bit-exact, ties across range boundaries broken by the lower key index."""
    wl = W.Workload("dec_int", S=64, T=40000, H=4, D=64, K=40, q_pos0=40000 - 64, seed=51, values="int")
    assert _splits(wl) > 1
    inp = W.generate(wl, "cuda")
    gpu = parity.run_gpu(wl, inp)
    parity.assert_exact(gpu, parity.oracle_rows(wl, inp, _rows(wl)), _rows(wl))


@pytest.mark.parametrize("wl", [
    W.Workload("dec_tok", S=8, T=60000, H=64, D=128, K=2048, q_pos0=60000 - 8, seed=52),
    W.Workload("dec_tok_short", S=5, T=5000, H=64, D=128, K=300, q_pos0=5000 - 5, seed=53),
    W.Workload("dec_fp8", S=4, T=40000, H=64, D=128, K=512, dtype="fp8", q_pos0=40000 - 4, seed=54),
    W.Workload("dec_pool", S=8, T=40000, H=32, D=128, K=256, visibility=W.POOLED, ratio=4,
               q_pos0=40000 - 8, seed=55),
    W.Workload("dec_csa", S=16, T=12000, H=64, D=128, K=512, visibility=W.COMPRESSED, ratio=4,
               q_pos0=4 * 12000 - 16, seed=56),
], ids=lambda w: w.name)
def test_decode_gaussian(cuda_ok, wl):
    assert _splits(wl) > 1
    inp = W.generate(wl, "cuda")
    gpu = parity.run_gpu(wl, inp)
    recall = parity.assert_tolerant(wl, gpu, parity.oracle_rows(wl, inp, _rows(wl)), _rows(wl))
    assert recall >= 0.9999


def test_decode_prune_bit_identical(cuda_ok):
    from head_weighted_relu_b200 import indexer as I
    wl = W.Workload("dec_prune", S=8, T=50000, H=64, D=128, K=1024, q_pos0=50000 - 8, seed=57, values="corr")
    assert _splits(wl) > 1
    inp = W.generate(wl, "cuda")
    args = dict(visibility=wl.visibility, ratio=wl.ratio, q_pos0=wl.q_pos0, q_scale=inp["q_scale"],
                k_scale=inp["k_scale"], pool_coef=inp["pool_coef"], with_scores=True)
    a = I.topk(inp["q"], inp["k"], inp["w"], wl.K, prune=False, **args)
    b = I.topk(inp["q"], inp["k"], inp["w"], wl.K, prune=True, **args)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x.nan_to_num(-7.0) if x.is_floating_point() else x,
                           y.nan_to_num(-7.0) if y.is_floating_point() else y)


def test_decode_matches_unsplit_shape(cuda_ok):
    """The same 4 query rows, once alone (split key ranges) and once inside a
    problem with enough query blocks to fill the GPU (one range per block):
    identical indices and lengths."""
    T = 30000
    big = W.Workload("dec_big", S=1024, T=T, H=64, D=128, K=512, q_pos0=T - 1024, seed=58)
    assert _splits(big) == 1
    inp = W.generate(big, "cuda")
    small = W.Workload("dec_small", S=4, T=T, H=64, D=128, K=512, q_pos0=T - 4, seed=58)
    assert _splits(small) > 1
    sub = {k: (v[-4:] if k in ("q", "w", "q_scale") and v is not None else v) for k, v in inp.items()}
    g_big = parity.run_gpu(big, inp, with_scores=False)
    g_small = parity.run_gpu(small, sub, with_scores=False)
    assert torch.equal(g_big[0][-4:], g_small[0]) and torch.equal(g_big[1][-4:], g_small[1])


@pytest.mark.parametrize("wl", [
    # a budget above the register-resident selection: the ranges and the merge
    # select on global memory
    W.Workload("dec_kbig", S=4, T=100000, H=64, D=128, K=4096, q_pos0=100000 - 4, seed=59),
    # 32 query rows per block (4 heads) over a key count that ends mid-tile
    W.Workload("dec_h4", S=40, T=33333, H=4, D=64, K=100, q_pos0=33333 - 40, seed=60),
], ids=lambda w: w.name)
def test_decode_edge_shapes(cuda_ok, wl):
    assert _splits(wl) > 1
    inp = W.generate(wl, "cuda")
    gpu = parity.run_gpu(wl, inp)
    recall = parity.assert_tolerant(wl, gpu, parity.oracle_rows(wl, inp, _rows(wl)), _rows(wl))
    assert recall >= 0.9999
