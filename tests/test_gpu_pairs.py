"""The adjacent-query-pair steps on the GPU against the oracle: the shared-index
count ("Adjacent-Query KV-Index Overlap in 256K DSA Training", §1, §3) and the
shared / left-only / right-only regions of a two-query cluster (same page,
§6.1, §6.4).  Both sides read the same seeded index rows, or rows each side
selected itself from the same integer-valued problem."""

import numpy as np
import pytest
import torch

import oracle
from head_weighted_relu_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


def _check_pairs(idx, ln, width, gpu_idx, gpu_len):
    """GPU pair steps on (gpu_idx, gpu_len) against the oracle on (idx, ln)."""
    from head_weighted_relu_b200 import indexer as I
    shared = I.pair_overlap(gpu_idx, gpu_len)
    sh, le, ri, counts = I.pair_regions(gpu_idx, gpu_len)
    torch.cuda.synchronize()
    ref_sh, ref_le, ref_ri, ref_counts = oracle.pair_regions(idx, ln, width)
    assert np.array_equal(shared.cpu().numpy(), oracle.pair_shared_counts(idx, ln))
    assert np.array_equal(counts.cpu().numpy(), ref_counts)
    assert np.array_equal(sh.cpu().numpy(), ref_sh)
    assert np.array_equal(le.cpu().numpy(), ref_le)
    assert np.array_equal(ri.cpu().numpy(), ref_ri)


@pytest.mark.parametrize("S,width,universe,seed", [
    (40, 64, 300, 1),        # several warps' worth of entries per row
    (37, 2048, 20000, 2),    # odd: the last row has no partner; full budget rows
    (12, 2051, 9000, 3),     # the pooled width
    (9, 1, 5, 4),            # one-slot rows
    (1, 16, 40, 5),          # no pair at all
])
def test_pair_steps_on_seeded_rows(cuda_ok, S, width, universe, seed):
    idx, ln = W.index_rows(S, width, universe, seed)
    _check_pairs(idx, ln, width, torch.from_numpy(idx).cuda(), torch.from_numpy(ln).cuda())


def test_pair_steps_on_indexer_rows(cuda_ok):
    """Integer inputs, so the indexer's rows equal the oracle's bit for bit;
    each side then runs its own pair steps on its own rows."""
    wl = W.Workload("pairs_int", S=256, T=900, H=4, D=64, K=64, q_pos0=900 - 256, seed=17, values="int")
    inp = W.generate(wl, "cuda")
    gpu = parity.run_gpu(wl, inp)
    rows = np.arange(wl.S, dtype=np.int64)
    ref = parity.oracle_rows(wl, inp, rows)
    parity.assert_exact(gpu, ref, rows)
    _check_pairs(ref["idx"], ref["len"], wl.K, gpu[0], gpu[1])


def test_pair_regions_rejects_bad_arguments(cuda_ok):
    from head_weighted_relu_b200 import indexer as I
    idx = torch.zeros((4, 8), dtype=torch.int32, device="cuda")
    ln = torch.zeros(4, dtype=torch.int32, device="cuda")
    out = [torch.empty((2, 8), dtype=torch.int32, device="cuda") for _ in range(3)]
    cnt = torch.empty((2, 3), dtype=torch.int32, device="cuda")
    with pytest.raises(I.IndexerError):
        I.indexer_pair_regions(idx, ln, -1, 8, *out, cnt)
    with pytest.raises(I.IndexerError):
        I.indexer_pair_regions(idx, ln, 4, 8, out[0], None, out[2], cnt)
