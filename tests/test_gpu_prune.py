"""The lossless pruning stage (INDEXER_FLAG_PRUNE): results bit-identical to
the run without it, on Gaussian inputs (where the certificate skips almost
nothing) and on structured inputs (near-identical heads, where it skips most
keys), and equal to the oracle."""

import numpy as np
import pytest
import torch

from head_weighted_relu_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


def _run(wl, inp, prune):
    from head_weighted_relu_b200 import indexer as I
    prob = I.make_problem(wl.S, wl.T, wl.H, wl.D, wl.K, wl.visibility, wl.ratio, wl.dtype,
                          wl.q_pos0, prune=prune)
    bufs = I.allocate(prob, "cuda", with_scores=True)
    out = I.topk(inp["q"], inp["k"], inp["w"], wl.K, visibility=wl.visibility, ratio=wl.ratio,
                 q_pos0=wl.q_pos0, q_scale=inp["q_scale"], k_scale=inp["k_scale"],
                 pool_coef=inp["pool_coef"], with_scores=True, buffers=bufs, prune=prune)
    torch.cuda.synchronize()
    counters = I.indexer_read_prune_counters(bufs[3])
    assert I.indexer_read_status(bufs[3]) == 0
    return out, counters


def _identical(a, b):
    for x, y in zip(a, b):
        if x.is_floating_point():
            assert torch.equal(x.nan_to_num(-7.0), y.nan_to_num(-7.0))
        else:
            assert torch.equal(x, y)


CASES = [
    W.Workload("gauss_bf16", S=1000, T=1000, H=64, D=128, K=128, seed=51),
    W.Workload("gauss_fp8", S=300, T=5000, H=64, D=128, K=512, dtype="fp8", q_pos0=4700, seed=52),
    W.Workload("gauss_pool_h32", S=1500, T=1500, H=32, D=128, K=128, visibility=W.POOLED, ratio=4, seed=53),
    W.Workload("corr_bf16", S=600, T=6000, H=64, D=128, K=256, q_pos0=5400, seed=54, values="corr"),
    W.Workload("corr_fp8", S=600, T=6000, H=64, D=128, K=256, dtype="fp8", q_pos0=5400, seed=55,
               values="corr"),
    W.Workload("corr_csa", S=4000, T=1000, H=64, D=128, K=64, visibility=W.COMPRESSED, ratio=4,
               seed=56, values="corr"),
]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_pruned_equals_unpruned_and_oracle(cuda_ok, wl):
    inp = W.generate(wl, "cuda")
    plain, c0 = _run(wl, inp, prune=False)
    pruned, (screened, bounded, skipped) = _run(wl, inp, prune=True)
    assert c0 == (0, 0, 0)
    _identical(plain, pruned)
    assert screened > 0 and skipped <= bounded <= screened
    print(f"{wl.name}: per-key pruning rate {bounded / screened:.3f}, "
          f"head sums skipped {skipped / screened:.3f}")
    if wl.values == "corr":
        assert bounded / screened > 0.2 and skipped > 0
    rows = np.arange(wl.S)
    parity.assert_tolerant(wl, pruned, parity.oracle_rows(wl, inp, rows), rows)


def test_pruning_rejected_below_32_heads(cuda_ok):
    from head_weighted_relu_b200 import indexer as I
    with pytest.raises(I.IndexerError) as e:
        I.indexer_workspace_bytes(I.make_problem(64, 64, 16, 128, 8, prune=True))
    assert e.value.status == 3


def test_full_size_long_1m_fp8_pruned_equals_unpruned(cuda_ok):
    """The 1M-key FP8 workload with and without the pruning stage: identical."""
    wl = W.WORKLOADS["long_1m_fp8"]
    inp = W.generate(wl, "cuda")
    plain, _ = _run(wl, inp, prune=False)
    pruned, (screened, bounded, skipped) = _run(wl, inp, prune=True)
    _identical(plain, pruned)
    print(f"long_1m_fp8: per-key pruning rate {bounded / max(screened, 1):.5f}, "
          f"head sums skipped {skipped / max(screened, 1):.5f}")
