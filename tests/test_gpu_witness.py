"""indexer_topk_witness: the query's starting threshold is the K-th lowered
exact score of its seed keys ("DoSA: Dots Sparse Attention", 核心方法, first
step; the decode remark in 实验结果), which must change no result.  Every
output is compared bit for bit with indexer_topk's on the same inputs, for
seeds that are ideal (the query's own selection), weak (random keys, another
query's selection), unusable (unsorted, invalid, too few), on the split
key-range path and the single-range path, every visibility mode, FP8 and the
pruning stage; one seeded run is also checked against the oracle."""

import numpy as np
import pytest
import torch

from head_weighted_relu_b200 import workloads as W
from tests import parity
from tests.test_gpu_decode import _splits

pytestmark = pytest.mark.gpu


def _problem(wl, prune=False):
    from head_weighted_relu_b200 import indexer as I
    return I.make_problem(wl.S, wl.T, wl.H, wl.D, wl.K, wl.visibility, wl.ratio, wl.dtype, wl.q_pos0, prune=prune)


def _plain(wl, inp, prune=False):
    from head_weighted_relu_b200 import indexer as I
    prob = _problem(wl, prune)
    idx, ln, sc, ws = I.allocate(prob, "cuda", with_scores=True)
    I.indexer_topk(prob, inp["q"], inp["k"], inp["w"], inp["q_scale"], inp["k_scale"], inp["pool_coef"],
                   idx, ln, sc, ws)
    torch.cuda.synchronize()
    assert I.indexer_read_status(ws) == 0
    return idx, ln, sc


def _seeded(wl, inp, seeds, prune=False):
    from head_weighted_relu_b200 import indexer as I
    prob = _problem(wl, prune)
    width = I.indexer_out_width(prob)
    idx = torch.full((wl.S, width), -7, dtype=torch.int32, device="cuda")
    ln = torch.full((wl.S,), -7, dtype=torch.int32, device="cuda")
    sc = torch.full((wl.S, width), -7.0, dtype=torch.float32, device="cuda")
    ws = torch.empty(I.indexer_witness_workspace_bytes(prob, seeds.shape[1]), dtype=torch.uint8, device="cuda")
    I.indexer_topk_witness(prob, inp["q"], inp["k"], inp["w"], inp["q_scale"], inp["k_scale"], inp["pool_coef"],
                           seeds.contiguous(), idx, ln, sc, ws)
    torch.cuda.synchronize()
    return (idx, ln, sc), I.indexer_read_status(ws)


def _assert_same(a, b):
    assert torch.equal(a[1], b[1])
    assert torch.equal(a[0], b[0])
    assert torch.equal(a[2].nan_to_num(-9.0), b[2].nan_to_num(-9.0))


def _seed_sets(wl, idx0):
    """Seed rows of every kind, built from the unseeded output idx0."""
    g = torch.Generator().manual_seed(wl.seed + 1000)
    S, width = idx0.shape
    base = idx0.cpu()
    shuffled = torch.stack([r[torch.randperm(width, generator=g)] for r in base])
    noisy = base.clone()
    noisy[torch.rand(noisy.shape, generator=g) < 0.1] = -1
    noisy[:, width // 2] = 2**31 - 1   # names no visible key: ignored
    # random visible keys, ascending, in the numbering of out_idx
    rand_rows = []
    for t in range(S):
        gpos = wl.q_pos0 + t
        hi = gpos + 1 if wl.visibility != W.COMPRESSED else (gpos + 1) // wl.ratio
        hi = min(hi, wl.T)
        n = min(width, hi)
        r = torch.sort(torch.randperm(hi, generator=g)[:n]).values.to(torch.int32)
        rand_rows.append(torch.cat([r, torch.full((width - n,), -1, dtype=torch.int32)]))
    return {
        "self": base,
        "adjacent": torch.roll(base, 1, 0),
        "shuffled": shuffled,
        "noisy": noisy,
        "random": torch.stack(rand_rows),
        "short": base[:, : width // 2],
        "none": base[:, :0],
    }


@pytest.mark.parametrize("wl", [
    W.Workload("wit_tok", S=16, T=60000, H=64, D=128, K=1024, q_pos0=60000 - 16, seed=91),
    W.Workload("wit_fp8", S=8, T=50000, H=64, D=128, K=512, dtype="fp8", q_pos0=50000 - 8, seed=92),
    W.Workload("wit_pool", S=8, T=50000, H=32, D=128, K=256, visibility=W.POOLED, ratio=4,
               q_pos0=50000 - 8, seed=93),
    W.Workload("wit_csa", S=16, T=12000, H=64, D=128, K=512, visibility=W.COMPRESSED, ratio=4,
               q_pos0=4 * 12000 - 16, seed=94),
    W.Workload("wit_int", S=16, T=20000, H=4, D=64, K=200, q_pos0=20000 - 16, seed=95, values="int"),
], ids=lambda w: w.name)
def test_witness_split_path_identical(cuda_ok, wl):
    assert _splits(wl) > 1
    inp = W.generate(wl, "cuda")
    ref = _plain(wl, inp)
    for name, seeds in _seed_sets(wl, ref[0]).items():
        out, status = _seeded(wl, inp, seeds.to("cuda"))
        assert status == 0, name
        _assert_same(out, ref)


@pytest.mark.parametrize("wl", [
    W.Workload("wit_prefill", S=700, T=700, H=64, D=128, K=64, seed=96),
    W.Workload("wit_prefill_int", S=900, T=900, H=4, D=64, K=40, seed=97, values="int"),
    W.Workload("wit_prefill_pool", S=1200, T=1200, H=32, D=128, K=64, visibility=W.POOLED, ratio=4, seed=98),
], ids=lambda w: w.name)
def test_witness_single_range_identical(cuda_ok, wl):
    assert _splits(wl) == 1
    inp = W.generate(wl, "cuda")
    ref = _plain(wl, inp)
    for name, seeds in _seed_sets(wl, ref[0]).items():
        out, status = _seeded(wl, inp, seeds.to("cuda"))
        assert status == 0, name
        _assert_same(out, ref)


def test_witness_with_pruning_identical(cuda_ok):
    """Seeds and the pruning certificate together (the certificate screens
    against the seeded threshold from the first tile)."""
    wl = W.Workload("wit_prune", S=8, T=50000, H=64, D=128, K=1024, q_pos0=50000 - 8, seed=99, values="corr")
    inp = W.generate(wl, "cuda")
    ref = _plain(wl, inp)
    out, status = _seeded(wl, inp, ref[0], prune=True)
    assert status == 0
    _assert_same(out, ref)


def test_witness_matches_oracle(cuda_ok):
    wl = W.Workload("wit_oracle", S=8, T=30000, H=64, D=128, K=512, q_pos0=30000 - 8, seed=100)
    inp = W.generate(wl, "cuda")
    ref = _plain(wl, inp)
    out, status = _seeded(wl, inp, torch.roll(ref[0], 1, 0))
    assert status == 0
    rows = np.arange(wl.S, dtype=np.int64)
    recall = parity.assert_tolerant(wl, out, parity.oracle_rows(wl, inp, rows), rows)
    assert recall >= 0.9999


def test_witness_rejects_bad_arguments(cuda_ok):
    from head_weighted_relu_b200 import indexer as I
    prob = I.make_problem(100, 100, 64, 128, 16)
    with pytest.raises(I.IndexerError):
        I.indexer_witness_workspace_bytes(prob, -1)
    inp = W.generate(W.Workload("wit_bad", S=100, T=100, H=64, D=128, K=16, seed=101), "cuda")
    seeds = torch.zeros((100, 8), dtype=torch.int32, device="cuda")
    idx = torch.empty((100, 16), dtype=torch.int32, device="cuda")
    ln = torch.empty((100,), dtype=torch.int32, device="cuda")
    small = torch.empty(I.indexer_witness_workspace_bytes(prob, 8) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(I.IndexerError) as e:
        I.indexer_topk_witness(prob, inp["q"], inp["k"], inp["w"], None, None, None, seeds, idx, ln, None, small)
    assert e.value.status == 2   # INDEXER_EWORKSPACE


def test_witness_threshold_against_oracle(cuda_ok):
    """The threshold the seed kernels compute (kept after the indexer's own
    workspace and the seed scores) is a lower bound of the oracle's exact K-th
    score over the row's distinct visible seeds, within twice the rounding
    margin of it; rows with fewer than K such seeds get no threshold (0)."""
    import oracle
    from head_weighted_relu_b200 import indexer as I
    wl = W.Workload("wit_thr", S=8, T=30000, H=64, D=128, K=512, q_pos0=30000 - 8, seed=102)
    inp = W.generate(wl, "cuda")
    ref = _plain(wl, inp)
    # even rows: their own selection (a tight threshold); odd rows: the row
    # above's (a loose one); the last row: half a row (too few seeds)
    seeds = torch.where((torch.arange(wl.S, device="cuda") % 2 == 0)[:, None], ref[0], torch.roll(ref[0], 1, 0))
    seeds[-1, wl.K // 2:] = -1
    seeds = seeds.contiguous()
    prob = _problem(wl)
    n = seeds.shape[1]
    ws = torch.empty(I.indexer_witness_workspace_bytes(prob, n), dtype=torch.uint8, device="cuda")
    idx = torch.empty_like(ref[0])
    ln = torch.empty_like(ref[1])
    I.indexer_topk_witness(prob, inp["q"], inp["k"], inp["w"], None, None, None, seeds, idx, ln, None, ws)
    torch.cuda.synchronize()
    assert I.indexer_read_status(ws) == 0
    off = I.indexer_workspace_bytes(prob) + (wl.S * n * 4 + 255) // 256 * 256
    thr = ws[off: off + 4 * wl.S].cpu().numpy().view(np.uint32)
    bits = np.where(thr & 0x80000000, thr & 0x7FFFFFFF, ~thr).astype(np.uint32)
    thr_f = bits.view(np.float32).astype(np.float64)

    rows = np.arange(wl.S, dtype=np.int64)
    h = parity.host_inputs(inp, rows)
    s_np = seeds.cpu().numpy()
    tau = oracle.witness_threshold(wl.problem(), h["q_rows"], h["k"], h["w_rows"], rows, s_np)
    keys = oracle.decode_keys_for(wl.problem(), h["k"])
    assert np.isnan(tau[-1]) and thr[-1] == 0
    for t in range(wl.S - 1):
        assert not np.isnan(tau[t])
        q_t = oracle.decode_bf16(h["q_rows"][t])
        amp = float(np.abs(h["w_rows"][t].astype(np.float64)) @ np.linalg.norm(q_t, axis=1))
        sk = oracle.witness_seed_keys(s_np[t], wl.q_pos0 + t, keys.shape[0], W.TOKEN, 1)
        kmax = float(np.linalg.norm(keys[sk], axis=1).max())
        margin = 2.0 ** -12 * kmax * amp
        assert thr_f[t] <= tau[t], (t, thr_f[t], tau[t])
        assert thr_f[t] >= tau[t] - 2 * margin - 1e-5 * abs(tau[t]), (t, thr_f[t], tau[t], margin)
