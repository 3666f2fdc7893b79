"""Packed-document batches on the GPU against the oracle: a query sees only its
own document, pooled keys never span a document boundary ("Module 06 — DSA &
KPool", §3 and "Ship it"), and indices come out as global positions."""

import numpy as np
import pytest
import torch

import oracle
from head_weighted_relu_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


def _run_docs(wl, inp, bounds):
    from head_weighted_relu_b200 import indexer as I
    prob = I.make_problem(wl.S, wl.T, wl.H, wl.D, wl.K, wl.visibility, wl.ratio, wl.dtype, wl.q_pos0)
    width = I.indexer_out_width(prob)
    idx = torch.full((wl.S, width), -7, dtype=torch.int32, device="cuda")
    ln = torch.full((wl.S,), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((wl.S, width), -7.0, dtype=torch.float32, device="cuda")
    ws = torch.empty(I.indexer_docs_workspace_bytes(prob, bounds), dtype=torch.uint8, device="cuda")
    I.indexer_topk_docs(prob, inp["q"], inp["k"], inp["w"], inp["q_scale"], inp["k_scale"], inp["pool_coef"],
                        bounds, idx, ln, sc, ws)
    torch.cuda.synchronize()
    assert I.indexer_read_status(ws) == 0
    return idx, ln, sc


def _oracle_docs(wl, inp, bounds):
    rows = np.arange(wl.S, dtype=np.int64)
    h = parity.host_inputs(inp, rows)
    idx, ln, sc, tau = oracle.topk_rows_docs(wl.problem(), h["q_rows"], h["k"], h["w_rows"], rows, bounds,
                                             q_scale_rows=h["q_scale_rows"], k_scale=h["k_scale"],
                                             pool_coef=h["pool_coef"])
    keys = oracle.decode_keys_for(dict(wl.problem(), visibility=W.TOKEN), h["k"], h["k_scale"])
    return dict(idx=idx, len=ln, score=sc, tau=tau, keys=keys, host=h)


@pytest.mark.parametrize("wl,bounds", [
    # one-token document; lengths off the tile grid
    (W.Workload("doc_tok", S=2600, T=2600, H=4, D=64, K=50, seed=81, values="int"), [0, 700, 701, 2001, 2600]),
    # documents that do not start on a multiple of the pool width
    (W.Workload("doc_pool", S=2000, T=2000, H=32, D=128, K=64, visibility=W.POOLED, ratio=4, seed=82,
                values="int"), [0, 501, 1203, 2000]),
    # compressed keys: documents start on whole compressed keys
    (W.Workload("doc_csa", S=2400, T=600, H=64, D=128, K=64, visibility=W.COMPRESSED, ratio=4, seed=83,
                values="int"), [0, 800, 804, 2400]),
], ids=lambda x: x.name if isinstance(x, W.Workload) else "")
def test_docs_integer_bit_exact(cuda_ok, wl, bounds):
    inp = W.generate(wl, "cuda")
    gpu = _run_docs(wl, inp, bounds)
    ref = _oracle_docs(wl, inp, bounds)
    parity.assert_exact(gpu, ref, np.arange(wl.S))


@pytest.mark.parametrize("wl,bounds", [
    (W.Workload("doc_gauss", S=3000, T=3000, H=64, D=128, K=256, seed=84), [0, 1000, 3000]),
    # a few queries at the end of a long document: the split key-range path
    (W.Workload("doc_decode", S=8, T=40000, H=64, D=128, K=512, q_pos0=40000 - 8, seed=85), [0, 9000, 40000]),
], ids=lambda x: x.name if isinstance(x, W.Workload) else "")
def test_docs_gaussian(cuda_ok, wl, bounds):
    inp = W.generate(wl, "cuda")
    gpu = _run_docs(wl, inp, bounds)
    ref = _oracle_docs(wl, inp, bounds)
    recall = parity.assert_tolerant(wl, gpu, ref, np.arange(wl.S))
    assert recall >= 0.9999
    # nothing from another document
    gi, gl = gpu[0].cpu().numpy(), gpu[1].cpu().numpy()
    for r in range(wl.S):
        g = wl.q_pos0 + r
        d = int(np.searchsorted(bounds, g, side="right")) - 1
        row = gi[r, : gl[r]]
        assert ((row >= bounds[d]) & (row <= g)).all()


def test_docs_reject_bad_bounds(cuda_ok):
    from head_weighted_relu_b200 import indexer as I
    prob = I.make_problem(100, 100, 64, 128, 16)
    for bad in ([0, 50, 50, 100], [0, 120], [10, 100], [0]):
        with pytest.raises(I.IndexerError):
            I.indexer_docs_workspace_bytes(prob, bad)
