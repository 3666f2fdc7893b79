"""The scoring kernel's wait-timeout path, exercised without a device fault:
with INDEXER_FLAG_TEST_WAIT_TIMEOUT every CTA's MMA issuer waits, after its
first tile, on a barrier nothing arrives at, for about a millisecond.  The
call must report the timeout in the status word (bit 0), and the device must
stay usable: the next ordinary call on the same workspace is checked against
the oracle."""

import numpy as np
import pytest
import torch

from head_weighted_relu_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wl", [
    # many query blocks: one work item per block
    W.Workload("tok", S=700, T=3000, H=64, D=128, K=128, q_pos0=2300, seed=61),
    # few query blocks: split key ranges and the merge step
    W.Workload("split", S=8, T=60000, H=64, D=128, K=256, q_pos0=60000 - 8, seed=62),
    W.Workload("fp8", S=500, T=2000, H=64, D=128, K=100, dtype="fp8", q_pos0=1500, seed=63),
], ids=lambda w: w.name)
def test_wait_timeout_reports_and_device_recovers(cuda_ok, wl):
    from head_weighted_relu_b200 import indexer as I
    inp = W.generate(wl, "cuda")
    args = (inp["q"], inp["k"], inp["w"], inp["q_scale"], inp["k_scale"], inp["pool_coef"])
    hook = I.make_problem(wl.S, wl.T, wl.H, wl.D, wl.K, wl.visibility, wl.ratio, wl.dtype, wl.q_pos0,
                          flags=I.FLAG_TEST_WAIT_TIMEOUT)
    plain = I.make_problem(wl.S, wl.T, wl.H, wl.D, wl.K, wl.visibility, wl.ratio, wl.dtype, wl.q_pos0)
    idx, ln, sc, ws = I.allocate(plain, "cuda", with_scores=True)
    assert I.indexer_workspace_bytes(hook) == ws.numel()
    for _ in range(2):   # twice: the path leaves nothing behind
        I.indexer_topk(hook, *args, idx, ln, sc, ws)
        assert I.indexer_read_status(ws) & 1 == 1
    I.indexer_topk(plain, *args, idx, ln, sc, ws)
    assert I.indexer_read_status(ws) == 0
    torch.cuda.synchronize()
    rows = np.arange(wl.S, dtype=np.int64)
    parity.assert_tolerant(wl, (idx, ln, sc), parity.oracle_rows(wl, inp, rows), rows)
