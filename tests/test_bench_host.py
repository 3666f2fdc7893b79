"""The benchmark's host arithmetic against closed forms: the visible (query,
key) pairs a step scores (the metric's unit), the FLOPs per pair, and the
algorithmic HBM bytes a step must move.  CPU only."""

import numpy as np
import pytest

import bench
from head_weighted_relu_b200 import workloads as W


def _pairs_closed_form(wl):
    """Token keys: query g sees g + 1 keys (capped at T).  Compressed keys and
    pools of m: query g sees floor((g + 1) / m) of them ("Module 06 — DSA &
    KPool", §3: a key or pool is visible once all its tokens are)."""
    g = np.arange(wl.q_pos0, wl.q_pos0 + wl.S, dtype=np.int64)
    if wl.visibility == W.TOKEN:
        return int(np.minimum(g + 1, wl.T).sum())
    cap = wl.T if wl.visibility == W.COMPRESSED else wl.T // wl.ratio
    return int(np.minimum((g + 1) // wl.ratio, cap).sum())


@pytest.mark.parametrize("name,pairs", [
    ("tiny_int_512", 512 * 513 // 2),
    ("dsa_prefill_64k", 65536 * 65537 // 2),
    # sum over t < S of floor((t + 1) / 4) = 2 M^2 - M with M = S / 4
    ("csa_m4_256k", 2 * 65536 ** 2 - 65536),
    ("pooled_tail_128k", 2 * 32768 ** 2 - 32768),
    # the last 16,384 of 1,048,576 positions, every earlier key visible
    ("long_1m_fp8", sum(range(1048576 - 16384 + 1, 1048576 + 1))),
])
def test_visible_pairs(name, pairs):
    wl = W.WORKLOADS[name]
    assert bench.visible_pairs(wl) == pairs
    assert bench.visible_pairs(wl) == _pairs_closed_form(wl)


def test_flops_per_pair():
    assert bench.flops_per_pair(W.WORKLOADS["dsa_prefill_64k"]) == 2 * 64 * 128
    assert bench.flops_per_pair(W.WORKLOADS["pooled_tail_128k"]) == 2 * 32 * 128


@pytest.mark.parametrize("name,gib", [
    # inputs read once plus index rows and lengths written once
    ("dsa_prefill_64k", 1.53), ("csa_m4_256k", 6.08), ("pooled_tail_128k", 2.05), ("long_1m_fp8", 0.387),
])
def test_algorithmic_hbm_bytes(name, gib):
    wl = W.WORKLOADS[name]
    h = bench.hbm_summary(wl, wl.S, 10.0, 6456.5)
    assert abs(h["algorithmic_bytes"] / 2 ** 30 - gib) < 0.01
    # spelled out for the token workload: q, k in bf16, w in fp32, idx and len in int32
    if name == "dsa_prefill_64k":
        S, T, H, D, K = wl.S, wl.T, wl.H, wl.D, wl.K
        assert h["algorithmic_bytes"] == S * H * D * 2 + T * D * 2 + S * H * 4 + S * K * 4 + S * 4
    assert h["materialised_scores_gib"] == pytest.approx(
        wl.S * (wl.T // wl.ratio if wl.visibility == W.POOLED else wl.T) * 4 / 2 ** 30)
