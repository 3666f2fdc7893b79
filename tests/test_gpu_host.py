"""indexer_topk_host -- the indexer on host buffers, with the query rows streamed
through the device in chunks -- gives exactly the results of indexer_topk on
device buffers (chunks start on query-block boundaries, so every query is
scored in the same block and column and selected the same way)."""

import pytest
import torch

from head_weighted_relu_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wl", [
    # three chunks of 4,096 rows and a ragged last one
    W.Workload("host_tok", S=9000, T=9000, H=64, D=128, K=512, seed=71),
    W.Workload("host_pool", S=9001, T=9001, H=32, D=128, K=256, visibility=W.POOLED, ratio=4, seed=72),
    W.Workload("host_fp8", S=4500, T=20000, H=64, D=128, K=300, dtype="fp8", q_pos0=20000 - 4500, seed=73),
    # a last chunk of 8 rows: the split key-range path inside the pipeline
    W.Workload("host_tail", S=8200, T=30000, H=64, D=128, K=256, q_pos0=30000 - 8200, seed=74),
    # one chunk only (a decode shape)
    W.Workload("host_dec", S=8, T=40000, H=64, D=128, K=512, q_pos0=40000 - 8, seed=75),
], ids=lambda w: w.name)
def test_host_pipeline_matches_device_call(cuda_ok, wl):
    from head_weighted_relu_b200 import indexer as I
    inp = W.generate(wl, "cuda")
    prob = I.make_problem(wl.S, wl.T, wl.H, wl.D, wl.K, wl.visibility, wl.ratio, wl.dtype, wl.q_pos0)
    ref_idx, ref_len, ref_sc, ws = I.allocate(prob, "cuda", with_scores=True)
    I.indexer_topk(prob, inp["q"], inp["k"], inp["w"], inp["q_scale"], inp["k_scale"], inp["pool_coef"],
                   ref_idx, ref_len, ref_sc, ws)
    torch.cuda.synchronize()

    host = {n: (t.cpu().pin_memory() if t is not None else None) for n, t in inp.items()}
    width = I.indexer_out_width(prob)
    idx = torch.full((wl.S, width), -7, dtype=torch.int32).pin_memory()
    ln = torch.full((wl.S,), -7, dtype=torch.int32).pin_memory()
    sc = torch.full((wl.S, width), -7.0, dtype=torch.float32).pin_memory()
    hws = torch.empty(I.indexer_host_workspace_bytes(prob), dtype=torch.uint8, device="cuda")
    for _ in range(2):   # the workspace and streams are reused by a second call
        I.indexer_topk_host(prob, host["q"], host["k"], host["w"], host["q_scale"], host["k_scale"],
                            host["pool_coef"], idx, ln, sc, hws)
        torch.cuda.synchronize()
        assert I.indexer_read_status(hws) == 0
        assert torch.equal(ln, ref_len.cpu())
        assert torch.equal(idx, ref_idx.cpu())
        assert torch.equal(sc.nan_to_num(-9.0), ref_sc.cpu().nan_to_num(-9.0))


def test_host_pipeline_rejects_small_workspace(cuda_ok):
    from head_weighted_relu_b200 import indexer as I
    prob = I.make_problem(100, 100, 64, 128, 16)
    q = torch.zeros((100, 64, 128), dtype=torch.bfloat16).pin_memory()
    k = torch.zeros((100, 128), dtype=torch.bfloat16).pin_memory()
    w = torch.zeros((100, 64), dtype=torch.float32).pin_memory()
    idx = torch.empty((100, 16), dtype=torch.int32).pin_memory()
    ln = torch.empty((100,), dtype=torch.int32).pin_memory()
    small = torch.empty(I.indexer_host_workspace_bytes(prob) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(I.IndexerError) as e:
        I.indexer_topk_host(prob, q, k, w, None, None, None, idx, ln, None, small)
    assert e.value.status == 2   # INDEXER_EWORKSPACE
