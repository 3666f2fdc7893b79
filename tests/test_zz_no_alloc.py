"""indexer_topk_noalloc: the entry point for callers that cannot allocate
device memory (allocator hooks, plugins whose framework owns all device
memory, programs that forbid allocation after start-up).  It must give the
same result as indexer_topk, call after call, although its scratch lives in
one fixed device array shared by every call.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""

import pytest
import torch

from head_weighted_relu_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


def _outputs(prob, device):
    from head_weighted_relu_b200 import indexer as I
    width = I.indexer_out_width(prob)
    return (torch.full((prob.S, width), -7, dtype=torch.int32, device=device),
            torch.full((prob.S,), -7, dtype=torch.int32, device=device),
            torch.full((prob.S, width), -7.0, dtype=torch.float32, device=device))


@pytest.mark.parametrize("wl", [
    W.Workload("tok", S=2000, T=2000, H=64, D=128, K=256, seed=41),
    W.Workload("pool", S=1500, T=1500, H=32, D=128, K=128, visibility=W.POOLED, ratio=4, seed=42),
    W.Workload("fp8", S=200, T=3000, H=64, D=128, K=300, dtype="fp8", q_pos0=2800, seed=43),
    # few query rows against many keys: key ranges split across CTAs, then merged
    W.Workload("decode", S=8, T=40000, H=64, D=128, K=512, q_pos0=40000 - 8, seed=44),
], ids=lambda w: w.name)
def test_noalloc_matches_workspace_entry_point(cuda_ok, wl):
    from head_weighted_relu_b200 import indexer as I
    inp = W.generate(wl, "cuda")
    q, k = inp["q"], inp["k"]
    prob = I.make_problem(wl.S, wl.T, wl.H, wl.D, wl.K, wl.visibility, wl.ratio, wl.dtype, wl.q_pos0)
    ref_idx, ref_len, ref_sc, ws = I.allocate(prob, "cuda", with_scores=True)
    I.indexer_topk(prob, q, k, inp["w"], inp["q_scale"], inp["k_scale"], inp["pool_coef"],
                   ref_idx, ref_len, ref_sc, ws)
    torch.cuda.synchronize()
    for _ in range(2):   # two calls in a row: the shared scratch keeps the last call's contents
        idx, ln, sc = _outputs(prob, "cuda")
        I.indexer_topk_noalloc(prob, q, k, inp["w"], inp["q_scale"], inp["k_scale"],
                               inp["pool_coef"], idx, ln, sc)
        torch.cuda.synchronize()
        assert torch.equal(ln, ref_len)
        assert torch.equal(idx, ref_idx)
        same = torch.isnan(sc) & torch.isnan(ref_sc)
        close = (sc - ref_sc).abs() <= parity.REL * ref_sc.abs().clamp_min(1e-30)
        assert bool((same | close).all())
        assert I.indexer_noalloc_read_status() == 0   # no wait timed out, no buffer overflowed


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_ok):
    from head_weighted_relu_b200 import indexer as I
    prob = I.make_problem(4096, 4096, 64, 128, 8192)    # needs far more than 64 MiB of scratch
    assert I.indexer_workspace_bytes(prob) > 64 * 2 ** 20
    q = torch.zeros((4096, 64, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((4096, 128), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((4096, 64), dtype=torch.float32, device="cuda")
    idx, ln, sc = _outputs(prob, "cuda")
    with pytest.raises(I.IndexerError) as e:
        I.indexer_topk_noalloc(prob, q, k, w, None, None, None, idx, ln, None)
    assert e.value.status == 2   # INDEXER_EWORKSPACE
    torch.cuda.synchronize()
    assert bool((ln == -7).all())   # nothing was launched
