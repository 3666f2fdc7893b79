"""Helpers shared by the GPU parity tests: run the CUDA path, run the oracle on
the same inputs, compare under the acceptance rules.

Acceptance (floating point inputs): index sets match except for keys whose
oracle score lies within rel * |tau_K| of the K-th oracle score; mean recall
>= 0.9999; every selected score within rel * max(|s_ref|, |tau_K|) of the
oracle's; rel = 1e-3.  Integer inputs: bit-exact indices, lengths and scores.
"""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from head_weighted_relu_b200 import workloads as W

REL = 1e-3


def run_gpu(wl, inp, with_scores=True):
    from head_weighted_relu_b200 import indexer as I
    out = I.topk(inp["q"], inp["k"], inp["w"], wl.K, visibility=wl.visibility,
                 ratio=wl.ratio, q_pos0=wl.q_pos0, q_scale=inp["q_scale"],
                 k_scale=inp["k_scale"], pool_coef=inp["pool_coef"], with_scores=with_scores)
    torch.cuda.synchronize()
    return out


def host_inputs(inp, rows):
    """Storage bits of the rows the oracle needs."""
    rows_t = torch.as_tensor(rows, device=inp["q"].device)
    h = dict(
        q_rows=W.to_host_bits(inp["q"].index_select(0, rows_t)),
        k=W.to_host_bits(inp["k"]),
        w_rows=W.to_host_bits(inp["w"].index_select(0, rows_t)),
        q_scale_rows=None if inp["q_scale"] is None else W.to_host_bits(inp["q_scale"].index_select(0, rows_t)),
        k_scale=W.to_host_bits(inp["k_scale"]),
        pool_coef=W.to_host_bits(inp["pool_coef"]),
    )
    return h


def oracle_rows(wl, inp, rows, threads=1):
    """The oracle on the given query rows; with threads > 1 the rows are spread
    over host threads, one row at a time per thread (NumPy's BLAS held to one
    thread per call).  Each row is the same plain computation either way."""
    h = host_inputs(inp, rows)
    prob = wl.problem()
    keys = oracle.decode_keys_for(prob, h["k"], h["k_scale"], h["pool_coef"])

    def run(sl):
        return oracle.topk_rows(prob, h["q_rows"][sl], h["k"], h["w_rows"][sl], rows[sl],
                                q_scale_rows=None if h["q_scale_rows"] is None else h["q_scale_rows"][sl],
                                k_scale=h["k_scale"], pool_coef=h["pool_coef"], keys_f64=keys)

    if threads <= 1:
        idx, ln, sc, tau = run(slice(None))
    else:
        import concurrent.futures as cf
        from threadpoolctl import threadpool_limits
        with threadpool_limits(1), cf.ThreadPoolExecutor(threads) as ex:
            parts = list(ex.map(run, [slice(i, i + 1) for i in range(len(rows))]))
        idx, ln, sc, tau = (np.concatenate([p[j] for p in parts]) for j in range(4))
    return dict(idx=idx, len=ln, score=sc, tau=tau, keys=keys, host=h)


def _q_row_f64(wl, h, r):
    if wl.dtype == "fp8":
        return oracle.decode_e4m3(h["q_rows"][r]) * np.asarray(h["q_scale_rows"][r], np.float64)[:, None]
    return oracle.decode_bf16(h["q_rows"][r])


def assert_exact(gpu, ref, rows):
    gi, gl, gs = (x.cpu().numpy() for x in gpu)
    gi, gl, gs = gi[rows], gl[rows], gs[rows]
    assert np.array_equal(gl, ref["len"]), np.nonzero(gl != ref["len"])
    assert np.array_equal(gi, ref["idx"]), np.nonzero((gi != ref["idx"]).any(axis=1))
    rs = ref["score"]
    both_nan = np.isnan(gs) & np.isnan(rs)
    assert np.all(both_nan | (gs.astype(np.float64) == rs)), "scores differ"


def assert_tolerant(wl, gpu, ref, rows, rel=REL, min_recall=0.9999, stats=None):
    """Index-set parity under the tolerance rule; returns the mean recall
    (and, given a dict `stats`, fills in the minimum recall and the largest
    score error relative to max(|s_ref|, |tau|))."""
    gi, gl, gs = (x.cpu().numpy() for x in gpu)
    gi, gl, gs = gi[rows], gl[rows], gs[rows]
    m = wl.ratio if wl.visibility == W.POOLED else 1
    recalls = []
    for r, t in enumerate(rows):
        L = int(ref["len"][r])
        assert int(gl[r]) == L, (t, int(gl[r]), L)
        assert np.all(gi[r, L:] == -1), t
        a = gi[r, :L]
        b = ref["idx"][r, :L]
        assert np.all(np.diff(a) > 0), ("not strictly ascending", t)
        tau = ref["tau"][r]
        g = wl.q_pos0 + int(t)
        if m > 1:  # pools: compare pool sets; tails must match exactly
            nt = (g + 1) % m
            assert np.array_equal(a[L - nt:], b[L - nt:]), ("tail", t)
            a_keys = np.unique(a[: L - nt] // m)
            b_keys = np.unique(b[: L - nt] // m)
            assert a_keys.size * m == L - nt
        else:
            a_keys, b_keys = a, b
        sa, sb = set(a_keys.tolist()), set(b_keys.tolist())
        diff = sa ^ sb
        if diff:
            assert not math.isnan(tau), ("sets differ below the budget", t, sorted(diff)[:8])
            q_t = _q_row_f64(wl, ref["host"], r)
            w_t = np.asarray(ref["host"]["w_rows"][r], np.float64)
            keys = np.array(sorted(diff), dtype=np.int64)
            s_ref = oracle.score_keys(q_t, w_t, ref["keys"][keys])
            near = np.abs(s_ref - tau) <= rel * abs(tau)
            assert near.all(), ("index sets differ away from the threshold", t, keys[~near][:8],
                                s_ref[~near][:8], tau)
        recalls.append(len(sa & sb) / len(sb) if sb else float(not sa))
        # scores of the selected keys
        sel = gs[r, : L - ((g + 1) % m if m > 1 else 0)].astype(np.float64)
        if sel.size:
            q_t = _q_row_f64(wl, ref["host"], r)
            w_t = np.asarray(ref["host"]["w_rows"][r], np.float64)
            ks = (a[: sel.size] // m).astype(np.int64)
            s_ref = oracle.score_keys(q_t, w_t, ref["keys"][ks])
            scale = np.maximum(np.abs(s_ref), abs(tau) if not math.isnan(tau) else np.abs(s_ref).max())
            err = np.abs(sel - s_ref)
            assert np.all(err <= rel * np.maximum(scale, 1e-30)), (t, err.max(), scale.min())
            if stats is not None:
                stats["max_rel_score_err"] = max(stats.get("max_rel_score_err", 0.0),
                                                 float(np.max(err / np.maximum(scale, 1e-30))))
    mean = float(np.mean(recalls)) if recalls else 1.0
    if stats is not None:
        stats["mean_recall"] = mean
        stats["min_recall"] = float(np.min(recalls)) if recalls else 1.0
        stats["rows"] = len(recalls)
        stats["rows_with_differences"] = int(sum(r < 1.0 for r in recalls))
    assert mean >= min_recall, mean
    return mean
