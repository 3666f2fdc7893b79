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


def _random_bounds(total, lo, hi, seed):
    """Document bounds of random lengths in [lo, hi] covering [0, total)."""
    rng = np.random.default_rng(seed)
    b = [0]
    while b[-1] < total:
        b.append(min(total, b[-1] + int(rng.integers(lo, hi + 1))))
    return b


# Batches with many query blocks run as one launch over a table of every
# document's blocks (the per-launch cost dominates short documents); these
# cover it for one-query (H = 64, 4), two-query (H = 32) and FP8 groups.
@pytest.mark.parametrize("wl,lengths", [
    (W.Workload("docs_many_h4", S=900, T=900, H=4, D=64, K=8, seed=89, values="int"), (1, 12)),
    (W.Workload("docs_many_h32", S=1200, T=1200, H=32, D=128, K=32, seed=87, values="int"), (1, 40)),
    (W.Workload("docs_many_csa", S=2000, T=500, H=64, D=128, K=16, visibility=W.COMPRESSED, ratio=4, seed=90,
                values="int"), (4, 60)),
], ids=lambda x: x.name if isinstance(x, W.Workload) else "")
def test_docs_one_launch_integer_bit_exact(cuda_ok, wl, lengths):
    key_tokens = wl.T * wl.ratio if wl.visibility == W.COMPRESSED else wl.T
    bounds = _random_bounds(key_tokens, *lengths, seed=wl.seed)
    if wl.visibility == W.COMPRESSED:   # documents start on whole compressed keys
        bounds = sorted(set([0] + [x // wl.ratio * wl.ratio for x in bounds[1:-1]] + [key_tokens]))
    inp = W.generate(wl, "cuda")
    gpu = _run_docs(wl, inp, bounds)
    ref = _oracle_docs(wl, inp, bounds)
    parity.assert_exact(gpu, ref, np.arange(wl.S))


def test_docs_one_launch_fp8(cuda_ok):
    wl = W.Workload("docs_fp8", S=800, T=800, H=64, D=128, K=64, dtype="fp8", seed=88)
    bounds = _random_bounds(wl.T, 10, 120, seed=88)
    inp = W.generate(wl, "cuda")
    gpu = _run_docs(wl, inp, bounds)
    ref = _oracle_docs(wl, inp, bounds)
    recall = parity.assert_tolerant(wl, gpu, ref, np.arange(wl.S))
    assert recall >= 0.9999
    gi, gl = gpu[0].cpu().numpy(), gpu[1].cpu().numpy()
    for r in range(wl.S):
        d = int(np.searchsorted(bounds, r, side="right")) - 1
        row = gi[r, : gl[r]]
        assert ((row >= bounds[d]) & (row <= r)).all()


def test_docs_reject_bad_bounds(cuda_ok):
    from head_weighted_relu_b200 import indexer as I
    prob = I.make_problem(100, 100, 64, 128, 16)
    for bad in ([0, 50, 50, 100], [0, 120], [10, 100], [0]):
        with pytest.raises(I.IndexerError):
            I.indexer_docs_workspace_bytes(prob, bad)


# ---------------------------------------------------------------------------
# Padded batches and the watch lengths in both batch forms
# ---------------------------------------------------------------------------

WATCH = [3, 4, 5, 7, 8, 9]   # "Module 06 — DSA & KPool", §3 (tests/golden/kpool_watch_lengths.txt)


def _run_padded(wl, inp, lens, stride):
    from head_weighted_relu_b200 import indexer as I
    prob = I.make_problem(wl.S, wl.T, wl.H, wl.D, wl.K, wl.visibility, wl.ratio, wl.dtype, wl.q_pos0)
    width = I.indexer_out_width(prob)
    idx = torch.full((wl.S, width), -7, dtype=torch.int32, device="cuda")
    ln = torch.full((wl.S,), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((wl.S, width), -7.0, dtype=torch.float32, device="cuda")
    ws = torch.empty(I.indexer_padded_workspace_bytes(prob, lens, stride), dtype=torch.uint8, device="cuda")
    I.indexer_topk_padded(prob, inp["q"], inp["k"], inp["w"], inp["q_scale"], inp["k_scale"], inp["pool_coef"],
                          lens, stride, idx, ln, sc, ws)
    torch.cuda.synchronize()
    assert I.indexer_read_status(ws) == 0
    return idx, ln, sc


def _oracle_padded(wl, inp, lens, stride):
    rows = np.arange(wl.S, dtype=np.int64)
    h = parity.host_inputs(inp, rows)
    idx, ln, sc, tau = oracle.topk_rows_padded(wl.problem(), h["q_rows"], h["k"], h["w_rows"], rows, lens, stride,
                                               q_scale_rows=h["q_scale_rows"], k_scale=h["k_scale"],
                                               pool_coef=h["pool_coef"])
    return dict(idx=idx, len=ln, score=sc, tau=tau, host=h)


@pytest.mark.parametrize("vis,ratio,K", [(W.TOKEN, 1, 4), (W.COMPRESSED, 4, 4), (W.POOLED, 4, 8)])
def test_watch_lengths_padded_and_packed(cuda_ok, vis, ratio, K):
    """The watch lengths as a padded batch (stride 12) and as a packed batch of
    documents; in the packed form a pool at a document's end would span the
    boundary if pools were formed on the global grid (documents start at 3, 7,
    12, 19 and 27).  Integer inputs: bit-exact against the oracle."""
    stride = 12
    S = stride * len(WATCH)
    T = S // ratio if vis == W.COMPRESSED else S
    wl = W.Workload("watch_pad", S=S, T=T, H=32, D=128, K=K, visibility=vis, ratio=ratio, seed=86 + vis,
                    values="int")
    inp = W.generate(wl, "cuda")
    gpu = _run_padded(wl, inp, WATCH, stride)
    ref = _oracle_padded(wl, inp, WATCH, stride)
    parity.assert_exact(gpu, ref, np.arange(S))
    gl = gpu[1].cpu().numpy()
    for b, L in enumerate(WATCH):
        assert (gl[b * stride + L:(b + 1) * stride] == 0).all()   # padding rows select nothing
    if vis == W.COMPRESSED:
        return   # packed documents of compressed keys must start on whole keys; the watch lengths do not
    bounds = np.concatenate([[0], np.cumsum(WATCH)]).tolist()
    n = bounds[-1]
    pw = W.Workload("watch_docs", S=n, T=n, H=32, D=128, K=K, visibility=vis, ratio=ratio, seed=96 + vis,
                    values="int")
    pin = W.generate(pw, "cuda")
    parity.assert_exact(_run_docs(pw, pin, bounds), _oracle_docs(pw, pin, bounds), np.arange(n))


def test_padded_gaussian_and_split_path(cuda_ok):
    """Longer padded sequences on Gaussian inputs, one of them empty and one a
    few rows long; a stride of 9,000 makes the short sequences take the split
    key-range path."""
    stride = 9000
    lens = [9000, 0, 5, 4097]
    S = stride * len(lens)
    wl = W.Workload("pad_gauss", S=S, T=S, H=64, D=128, K=256, seed=87)
    inp = W.generate(wl, "cuda")
    gpu = _run_padded(wl, inp, lens, stride)
    rows = np.concatenate([np.arange(0, 600), np.arange(8990, 9010), np.arange(18000, 18010),
                           np.arange(27000, 27000 + 4100)])
    h = parity.host_inputs(inp, rows)
    idx, ln, sc, tau = oracle.topk_rows_padded(wl.problem(), h["q_rows"], h["k"], h["w_rows"], rows, lens, stride)
    ref = dict(idx=idx, len=ln, score=sc, tau=tau, host=h,
               keys=oracle.decode_keys_for(wl.problem(), h["k"]))
    parity.assert_tolerant(wl, gpu, ref, rows)


def test_padded_rejects_bad_shapes(cuda_ok):
    from head_weighted_relu_b200 import indexer as I
    ok = I.make_problem(24, 24, 64, 128, 8)
    assert I.indexer_padded_workspace_bytes(ok, [12, 5], 12) >= 256
    for prob, lens, stride in ((ok, [13, 5], 12), (ok, [12, 5], 11), (I.make_problem(24, 24, 64, 128, 8, q_pos0=0), [12], 12),
                               (I.make_problem(24, 5, 64, 128, 8, I.COMPRESSED, 4), [12, 12], 12)):
        with pytest.raises(I.IndexerError):
            I.indexer_padded_workspace_bytes(prob, lens, stride)
