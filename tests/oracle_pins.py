"""Pins that tie the CPU oracle to facts outside itself.

Each pin takes the oracle module as an argument (so the mutation test can run
the same pins against a copy of the oracle with a planted mistake) and raises
AssertionError when the oracle disagrees with:
  * values the source pages print (tests/golden/*.txt, each with its citation),
  * a hand-worked example (tests/golden/hand_worked_scores.json),
  * brute force on tiny inputs (Python integers, subset enumeration),
  * closed forms and invariants of the definitions,
  * library routines for the storage formats (torch's float8/bfloat16 casts,
    Python sets, exact rationals).
"""

from __future__ import annotations

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                out.append([int(x) for x in line.split()])
    return out


def _bf16_bits_of_ints(a) -> np.ndarray:
    """Small integers -> bf16 bit patterns via torch (exact for |x| <= 256)."""
    t = torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _problem(S, T, H, D, K, vis=0, ratio=1, dtype="bf16", q_pos0=0):
    return dict(S=S, T=T, H=H, D=D, K=K, visibility=vis, ratio=ratio,
                dtype=dtype, q_pos0=q_pos0)


def _beats(a, b):
    """(score, index) a is ranked above b: higher score, then lower index."""
    return a[0] > b[0] or (a[0] == b[0] and a[1] < b[1])


# ----------------------------------------------------------------------------
# score arithmetic
# ----------------------------------------------------------------------------

def pin_hand_worked(O):
    with open(os.path.join(GOLDEN, "hand_worked_scores.json")) as f:
        ex = json.load(f)
    q = np.array(ex["q"], dtype=np.float64)
    w = np.array(ex["w"], dtype=np.float64)
    keys = np.array(ex["keys"], dtype=np.float64)
    s = O.score_keys(q, w, keys)
    assert s.tolist() == [float(x) for x in ex["scores"]], s
    qb = _bf16_bits_of_ints(q)[None]
    kb = _bf16_bits_of_ints(keys)
    for case in ex["cases"]:
        g, K = case["g"], case["K"]
        prob = _problem(S=g + 1, T=len(keys), H=ex["H"], D=ex["D"], K=K)
        idx, ln, sc, tau = O.topk_rows(prob, qb, kb, w[None].astype(np.float32), [g])
        assert int(ln[0]) == len(case["idx"]), (case, ln)
        assert idx[0, : ln[0]].tolist() == case["idx"], (case, idx)
        assert (idx[0, ln[0]:] == -1).all()


def pin_integer_bruteforce(O):
    rng = np.random.default_rng(7)
    for trial in range(6):
        H, D, n = int(rng.integers(1, 5)), int(rng.integers(1, 9)), 16
        q = rng.integers(-3, 4, size=(H, D))
        w = rng.integers(-2, 3, size=H)
        keys = rng.integers(-3, 4, size=(n, D))
        expect = []
        for i in range(n):
            tot = 0
            for h in range(H):
                dot = 0
                for d in range(D):
                    dot += int(q[h, d]) * int(keys[i, d])
                tot += int(w[h]) * max(dot, 0)
            expect.append(tot)
        got = O.score_keys(q.astype(np.float64), w.astype(np.float64), keys.astype(np.float64))
        assert got.tolist() == [float(x) for x in expect], (trial, got, expect)


def pin_score_properties(O):
    rng = np.random.default_rng(11)
    H, D, n = 5, 16, 40
    q = rng.standard_normal((H, D))
    w = rng.standard_normal(H)
    keys = rng.standard_normal((n, D))
    s = O.score_keys(q, w, keys)
    # positive homogeneity in the key and in the weights
    assert np.allclose(O.score_keys(q, w, 2.0 * keys), 2.0 * s, rtol=1e-12, atol=1e-12)
    assert np.allclose(O.score_keys(q, -w, keys), -s, rtol=1e-12, atol=1e-12)
    # the score is linear in w: s(w1 + w2) = s(w1) + s(w2)
    w2 = rng.standard_normal(H)
    assert np.allclose(O.score_keys(q, w + w2, keys), s + O.score_keys(q, w2, keys), rtol=1e-10, atol=1e-10)
    # heads are interchangeable when q rows and weights move together
    perm = rng.permutation(H)
    assert np.allclose(O.score_keys(q[perm], w[perm], keys), s, rtol=1e-12, atol=1e-12)
    # one head with weight 1: s = max(0, q.k); a key opposite to q scores 0
    e0 = np.zeros(H)
    e0[0] = 1.0
    s0 = O.score_keys(q, e0, keys)
    assert np.allclose(s0, np.maximum(keys @ q[0], 0.0), rtol=1e-12, atol=1e-12)
    assert O.score_keys(q, e0, -q[:1])[0] == 0.0
    # a negative weight on an active head lowers the score
    e1 = np.zeros(H)
    e1[1] = -1.0
    assert O.score_keys(q, e1, q[1:2])[0] < 0


# ----------------------------------------------------------------------------
# selection
# ----------------------------------------------------------------------------

def pin_selection_bruteforce(O):
    rng = np.random.default_rng(3)
    for trial in range(60):
        n = int(rng.integers(1, 11))
        K = int(rng.integers(1, 6))
        s = rng.integers(-2, 3, size=n).astype(np.float64)  # many ties
        if trial % 3 == 0:
            s = -s * 0.0  # all zero, some -0.0
        keys = np.arange(n, dtype=np.int64)
        m = min(K, n)
        winners = []
        for sub in itertools.combinations(range(n), m):
            rest = [i for i in range(n) if i not in sub]
            if all(_beats((s[a], a), (s[b], b)) for a in sub for b in rest):
                winners.append(sub)
        assert len(winners) == 1, (s, K, winners)
        sel, ssel, tau = O.select_topk(s + 0.0, keys, K)
        assert sel.tolist() == list(winners[0]), (trial, s, K, sel, winners)
        assert ssel.tolist() == [s[i] + 0.0 for i in winners[0]]


def pin_selection_dominance(O):
    rng = np.random.default_rng(5)
    n, K = 400, 57
    s = np.round(rng.standard_normal(n) * 4) / 2  # ties on a 0.5 grid
    keys = np.arange(n, dtype=np.int64) * 3 + 1     # ascending, not 0..n-1
    sel, ssel, tau = O.select_topk(s, keys, K)
    assert sel.size == K and np.all(np.diff(sel) > 0)
    chosen = set(sel.tolist())
    pos = {int(k): i for i, k in enumerate(keys)}
    ins = [(s[pos[k]], k) for k in chosen]
    outs = [(s[i], int(keys[i])) for i in range(n) if int(keys[i]) not in chosen]
    for a in ins:
        for b in outs:
            assert _beats(a, b), (a, b)
    kth = sorted(ins, key=lambda x: (-x[0], x[1]))[-1]
    assert tau == kth[0]


def pin_chunked_equals_materialised(O):
    """StreamIndex (arXiv 2605.02568, abstract): a chunked partition-merge top-K
    must reproduce the materialised result.  The chunked side here is an
    independent tuple sort: per chunk keep the best K, then merge."""
    rng = np.random.default_rng(9)
    for trial in range(8):
        n = int(rng.integers(50, 600))
        K = int(rng.integers(1, 80))
        chunk = int(rng.integers(7, 130))
        s = np.round(rng.standard_normal(n) * 3)  # integer scores: ties
        keys = np.arange(n, dtype=np.int64)
        kept = []
        for c0 in range(0, n, chunk):
            part = [(-s[i], i) for i in range(c0, min(n, c0 + chunk))]
            kept.extend(sorted(part)[:K])
            kept = sorted(kept)[:K]
        expect = sorted(i for _, i in kept)
        sel, _, _ = O.select_topk(s, keys, K)
        assert sel.tolist() == expect, (trial, n, K, chunk)


def pin_row_invariants(O):
    rng = np.random.default_rng(21)
    H, D, T, K = 3, 8, 300, 40
    qb = _bf16_bits_of_ints(rng.integers(-3, 4, size=(T, H, D)))
    kb = _bf16_bits_of_ints(rng.integers(-3, 4, size=(T, D)))
    w = rng.integers(-2, 3, size=(T, H)).astype(np.float32)
    rows = np.arange(0, T, 7)
    for vis, ratio in ((0, 1), (1, 4), (2, 4)):
        prob = _problem(S=T, T=T, H=H, D=D, K=K, vis=vis, ratio=ratio)
        idx, ln, sc, tau = O.topk_rows(prob, qb[rows], kb, w[rows], rows,
                                       pool_coef=_bf16_bits_of_ints(np.ones((ratio, D))))
        width = O.out_width(K, vis, ratio)
        assert idx.shape == (rows.size, width)
        for r, t in enumerate(rows):
            g = int(t)
            row = idx[r, : ln[r]]
            assert np.all(np.diff(row) > 0), (vis, t, row)
            assert np.all(idx[r, ln[r]:] == -1)
            if vis == 0:
                assert ln[r] == min(K, g + 1)
                assert row.size == 0 or row[-1] <= g
            elif vis == 1:
                nv = min((g + 1) // ratio, T)
                assert ln[r] == min(K, nv)
                assert np.all(ratio * row + ratio - 1 <= g)
            else:
                nc = (g + 1) // ratio
                assert ln[r] == ratio * min(K // ratio, nc) + (g + 1) % ratio
                assert np.all(row <= g)


def pin_prefix_closed_form(O):
    """Token rows whose whole prefix fits in the budget select exactly 0..g."""
    rng = np.random.default_rng(4)
    H, D, T, K = 2, 4, 64, 16
    qb = _bf16_bits_of_ints(rng.integers(-3, 4, size=(T, H, D)))
    kb = _bf16_bits_of_ints(rng.integers(-3, 4, size=(T, D)))
    w = rng.integers(-2, 3, size=(T, H)).astype(np.float32)
    rows = np.arange(K)
    idx, ln, _, _ = O.topk_rows(_problem(T, T, H, D, K), qb[rows], kb, w[rows], rows)
    for g in range(K):
        assert idx[g, : ln[g]].tolist() == list(range(g + 1))


# ----------------------------------------------------------------------------
# visibility, pooling, slots
# ----------------------------------------------------------------------------

def pin_visibility_closed_forms(O):
    T = 50
    for g in range(0, 230):
        assert O.visible_keys(g, T, O.TOKEN, 1).tolist() == list(range(min(g + 1, T)))
        for m in (1, 2, 4, 7):
            v = O.visible_keys(g, T, O.COMPRESSED, m)
            assert v.tolist() == list(range(min((g + 1) // m, T))), (g, m)
            lit = [p for p in range(T) if all(m * p + j <= g for j in range(m))]
            assert O.visible_keys(g, T, O.POOLED, m).tolist() == lit, (g, m)


def pin_watch_lengths(O):
    for L, pools, tail in _rows("kpool_watch_lengths.txt"):
        g = L - 1
        assert O.visible_keys(g, 1000, O.POOLED, 4).size == pools, L
        assert O.incomplete_tail(g, 4).size == tail, L
        assert O.incomplete_tail(g, 4).tolist() == list(range(4 * pools, g + 1))
        # through the full row path, with a budget larger than the history
        D = 2
        kb = _bf16_bits_of_ints(np.ones((16, D)))
        qb = _bf16_bits_of_ints(np.ones((1, 1, D)))
        prob = _problem(S=g + 1, T=16, H=1, D=D, K=8, vis=O.POOLED, ratio=4)
        idx, ln, _, _ = O.topk_rows(prob, qb, kb, np.ones((1, 1), np.float32), [g],
                                    pool_coef=_bf16_bits_of_ints(np.ones((4, D))))
        assert int(ln[0]) == 4 * pools + tail
        assert idx[0, : ln[0]].tolist() == list(range(L)), (L, idx)


def pin_slot_count(O):
    budget, width, pools, slots = _rows("kpool_slots.txt")[0]
    assert O.out_width(budget, O.POOLED, width) == slots
    assert budget // width == pools
    # a row that fills every slot: >= 512 complete pools and a 3-token tail
    D, T = 2, 4 * 600
    g = 4 * 515 + 2
    kb = _bf16_bits_of_ints(np.ones((T, D)))
    qb = _bf16_bits_of_ints(np.ones((1, 1, D)))
    prob = _problem(S=g + 1, T=T, H=1, D=D, K=budget, vis=O.POOLED, ratio=width)
    idx, ln, _, _ = O.topk_rows(prob, qb, kb, np.ones((1, 1), np.float32), [g],
                                pool_coef=_bf16_bits_of_ints(np.ones((width, D))))
    assert idx.shape[1] == slots and int(ln[0]) == slots


def pin_pooled_keys(O):
    rng = np.random.default_rng(13)
    T, D, m = 40, 6, 4
    kb = _bf16_bits_of_ints(rng.integers(-3, 4, size=(T, D)))
    # one-hot coefficients pick one constituent exactly
    for j in range(m):
        c = np.zeros((m, D))
        c[j] = 1.0
        kp = O.pooled_keys(kb, _bf16_bits_of_ints(c), m)
        assert (kp == kb[j::m][: T // m]).all(), j
    # unit coefficients: integer sums, exact
    ints = rng.integers(-3, 4, size=(T, D))
    kp = O.pooled_keys(_bf16_bits_of_ints(ints), _bf16_bits_of_ints(np.ones((m, D))), m)
    expect = ints.reshape(T // m, m, D).sum(axis=1)
    assert (kp == _bf16_bits_of_ints(expect)).all()
    # general values against exact rationals and a nearest-value search
    kf = torch.randn(T, D, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    cf = (torch.rand(m, D, generator=torch.Generator().manual_seed(2)) * 0.5).to(torch.bfloat16)
    kbits = kf.view(torch.int16).numpy().view(np.uint16)
    cbits = cf.view(torch.int16).numpy().view(np.uint16)
    kp = O.pooled_keys(kbits, cbits, m)
    kv, cv = kf.float().numpy(), cf.float().numpy()
    for p in range(T // m):
        for d in range(D):
            exact = sum(Fraction(float(kv[m * p + j, d])) * Fraction(float(cv[j, d])) for j in range(m))
            assert int(kp[p, d]) == _nearest_bf16_bits(exact), (p, d)


def pooled_rounding_cases():
    """Columns of tests/golden/pooled_rounding_cases.txt: (k [4] values,
    c [4] values, expected bfloat16 bits), values as exact Fractions."""
    out = []
    with open(os.path.join(GOLDEN, "pooled_rounding_cases.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            nums = [int(x) for x in parts[:16]]
            vals = [Fraction(nums[2 * i]) * Fraction(2) ** nums[2 * i + 1] for i in range(8)]
            out.append((vals[:4], vals[4:], int(parts[16], 0)))
    return out


def _bf16_bits_of_fractions(vals) -> np.ndarray:
    """Exact bfloat16 values (as Fractions) -> bit patterns, through torch."""
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64).to(torch.bfloat16)
    back = t.double().numpy()
    assert all(Fraction(float(b)) == v for b, v in zip(back, vals)), "not a bfloat16 value"
    return t.view(torch.int16).numpy().view(np.uint16)


def wide_pool_columns(n_cols: int, seed: int):
    """Random pool columns (k [n_cols pools of 4 tokens, 1 channel] and c
    [4, n_cols]) whose products span up to 2^80 in magnitude, so that most
    binary64 running sums are inexact.  Returns bf16 bits k [4 * n, 1] laid
    out as n pools of one channel, and c [4, 1] per column as a list."""
    rng = np.random.default_rng(seed)
    mant = rng.integers(1, 256, size=(n_cols, 8)) * rng.choice([-1, 1], size=(n_cols, 8))
    expo = rng.integers(-40, 41, size=(n_cols, 8))
    return [[Fraction(int(m)) * Fraction(2) ** int(e) for m, e in zip(mant[i], expo[i])] for i in range(n_cols)]


def pin_pooled_keys_inexact_sums(O):
    """Pool keys whose binary64 running sum is inexact ("Module 06 — DSA &
    KPool", §2; one RNE rounding of the exact sum): the hand-worked columns of
    tests/golden/pooled_rounding_cases.txt (ties hidden by cancelling terms,
    subnormal and overflowing results, a cancellation a double-double
    accumulation gets wrong) and random columns with exponent spreads up to
    2^80, each against the nearest bfloat16 of the exact rational sum."""
    cases = pooled_rounding_cases()
    # one column per case: c varies by channel, so each case gets its own channel
    D = len(cases)
    k = np.zeros((4, D), dtype=np.uint16)
    c = np.zeros((4, D), dtype=np.uint16)
    for d, (kv, cv, _) in enumerate(cases):
        k[:, d] = _bf16_bits_of_fractions(kv)
        c[:, d] = _bf16_bits_of_fractions(cv)
    got = O.pooled_keys(k, c, 4)
    assert got.shape == (1, D)
    for d, (kv, cv, want) in enumerate(cases):
        exact = sum(a * b for a, b in zip(kv, cv))
        assert _nearest_bf16_bits(exact) == want, (d, hex(want))
        assert int(got[0, d]) == want, (d, hex(int(got[0, d])), hex(want))
    # random wide columns: every pool of a channel shares that channel's c
    cols = wide_pool_columns(240, seed=19)
    n_pools, D = 6, len(cols) // 6
    k = np.zeros((4 * n_pools, D), dtype=np.uint16)
    c = np.zeros((4, D), dtype=np.uint16)
    inexact = 0
    for d in range(D):
        c[:, d] = _bf16_bits_of_fractions(cols[d * n_pools][4:])
        for p in range(n_pools):
            k[4 * p: 4 * p + 4, d] = _bf16_bits_of_fractions(cols[d * n_pools + p][:4])
    got = O.pooled_keys(k, c, 4)
    kf = [[Fraction(float(x)) for x in row] for row in O.decode_bf16(k).tolist()]
    cf = [[Fraction(float(x)) for x in row] for row in O.decode_bf16(c).tolist()]
    for p in range(n_pools):
        for d in range(D):
            exact = sum(kf[4 * p + j][d] * cf[j][d] for j in range(4))
            fsum = 0.0
            for j in range(4):
                fsum += float(kf[4 * p + j][d] * cf[j][d])
            inexact += Fraction(fsum) != exact
            assert int(got[p, d]) == _nearest_bf16_bits(exact), (p, d)
    assert inexact >= 60, inexact   # most columns exercise the exact-sum fallback


_LADDER = []


def _bf16_ladder():
    """Every non-negative finite bfloat16 value as a Fraction, in pattern order,
    then 2^128 for the infinity pattern (built once)."""
    if not _LADDER:
        vals = torch.arange(0, 0x7F80, dtype=torch.int32).to(torch.int16).view(torch.bfloat16).double().numpy()
        _LADDER.extend(Fraction(float(x)) for x in vals)
        _LADDER.append(Fraction(2) ** 128)
    return _LADDER


def _nearest_bf16_bits(v: Fraction) -> int:
    """Nearest bfloat16 to an exact rational (ties to the even pattern), found
    by bisection over the ordered positive bit patterns, decoded by torch.
    The infinity pattern 0x7F80 stands for 2^128 (IEEE overflow under
    round-to-nearest: at or above the largest finite value plus half its
    spacing the result is infinite)."""
    if v == 0:
        return 0
    sign = 0x8000 if v < 0 else 0
    a = abs(v)
    pats = _bf16_ladder()
    if a >= pats[-1]:
        return sign | 0x7F80
    lo, hi = 0, len(pats) - 1
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if pats[mid] <= a:
            lo = mid
        else:
            hi = mid
    dl = a - pats[lo]
    dh = pats[hi] - a
    if dl < dh or (dl == dh and lo % 2 == 0):
        return sign | lo
    return sign | hi


# ----------------------------------------------------------------------------
# storage formats against library casts
# ----------------------------------------------------------------------------

def pin_e4m3_decoder(O):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.decode_e4m3(codes)
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.all(both_nan | (ref == got)), np.nonzero(~(both_nan | (ref == got)))
    assert np.nanmax(got) == 448.0


def pin_bf16_codec(O):
    rng = np.random.default_rng(17)
    bits = rng.integers(0, 1 << 16, size=20000).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]  # finite patterns
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.decode_bf16(bits), ref)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),            # subnormal
        np.array([3.3e38, -3.39e38, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 0.0, -0.0], np.float32),
    ])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.round_to_bf16_bits(x.astype(np.float64))
    assert np.array_equal(got, ref), np.nonzero(got != ref)
    # binary64 inputs carrying bits beyond binary32 (sticky bits matter)
    for v in (1.0 + 2 ** -8 + 2 ** -40, 1.0 + 2 ** -8 - 2 ** -40, -(3.0 + 2 ** -7 + 2 ** -50), 12345.678901234):
        assert int(O.round_to_bf16_bits(np.array([v]))[0]) == _nearest_bf16_bits(Fraction(v)), v


# ----------------------------------------------------------------------------
# adjacent-pair overlap
# ----------------------------------------------------------------------------

def pin_pair_overlap(O):
    rng = np.random.default_rng(23)
    S, W = 40, 30
    idx = np.full((S, W), -1, dtype=np.int32)
    ln = np.zeros(S, dtype=np.int32)
    for r in range(S):
        n = int(rng.integers(0, W + 1))
        row = np.sort(rng.choice(60, size=n, replace=False))
        idx[r, :n] = row
        ln[r] = n
    got = O.pair_shared_counts(idx, ln)
    assert got.size == S // 2
    for p in range(S // 2):
        a = set(idx[2 * p, : ln[2 * p]].tolist())
        b = set(idx[2 * p + 1, : ln[2 * p + 1]].tolist())
        assert got[p] == len(a & b), p
    # nested causal prefixes: the even row is contained in the odd row
    idx2 = np.full((6, 8), -1, np.int32)
    ln2 = np.array([1, 2, 3, 4, 5, 6], np.int32)
    for r in range(6):
        idx2[r, : r + 1] = np.arange(r + 1)
    assert O.pair_shared_counts(idx2, ln2).tolist() == [1, 3, 5]


def pin_pair_regions(O):
    """Shared / left-only / right-only regions of a pair ("Adjacent-Query
    KV-Index Overlap in 256K DSA Training", §6.1, §6.4): a hand example, then
    properties on random rows -- shared + left rebuilds the left row, shared +
    right the right row, the three regions are disjoint and ascending, and the
    shared length equals the overlap count computed by the independent
    sort-and-count method."""
    idx = np.array([[1, 3, 5, 7, -1], [3, 4, 7, 9, 11]], np.int32)
    sh, le, ri, c = O.pair_regions(idx, np.array([4, 5], np.int32), 5)
    assert sh[0].tolist() == [3, 7, -1, -1, -1]
    assert le[0].tolist() == [1, 5, -1, -1, -1]
    assert ri[0].tolist() == [4, 9, 11, -1, -1]
    assert c[0].tolist() == [2, 2, 3]
    rng = np.random.default_rng(31)
    S, W = 41, 24   # odd: the last row has no partner
    idx = np.full((S, W), -1, dtype=np.int32)
    ln = np.zeros(S, dtype=np.int32)
    for r in range(S):
        n = int(rng.integers(0, W + 1))
        idx[r, :n] = np.sort(rng.choice(40, size=n, replace=False))
        ln[r] = n
    idx[2, : ln[3]] = idx[3, : ln[3]]   # one pair of identical rows
    ln[2] = ln[3]
    sh, le, ri, c = O.pair_regions(idx, ln, W)
    assert sh.shape == (S // 2, W) and c.shape == (S // 2, 3)
    assert np.array_equal(c[:, 0], O.pair_shared_counts(idx, ln))
    for p in range(S // 2):
        a = idx[2 * p, : ln[2 * p]].tolist()
        b = idx[2 * p + 1, : ln[2 * p + 1]].tolist()
        ns, nl, nr = c[p].tolist()
        s_, l_, r_ = sh[p, :ns].tolist(), le[p, :nl].tolist(), ri[p, :nr].tolist()
        assert sorted(s_ + l_) == a and sorted(s_ + r_) == b, p
        assert not (set(s_) & set(l_)) and not (set(s_) & set(r_)) and not (set(l_) & set(r_)), p
        for region in (s_, l_, r_):
            assert region == sorted(region)
        assert (sh[p, ns:] == -1).all() and (le[p, nl:] == -1).all() and (ri[p, nr:] == -1).all()
    assert c[1, 1] == 0 and c[1, 2] == 0   # identical rows: nothing unique


def pin_documents(O):
    """Packed documents ("Module 06 — DSA & KPool", §3 and "Ship it"): one
    document covering everything is the plain indexer; for token keys the
    output equals a brute-force top-K of the full score row with every key
    outside [document start, g] excluded; pooled output never leaves the
    query's document, comes in whole pools aligned to the document start, and
    ends with the document-relative incomplete tail."""
    rng = np.random.default_rng(37)
    H, D, T = 3, 8, 40
    qb = _bf16_bits_of_ints(rng.integers(-3, 4, size=(T, H, D)))
    kb = _bf16_bits_of_ints(rng.integers(-3, 4, size=(T, D)))
    w = rng.integers(-2, 3, size=(T, H)).astype(np.float32)
    rows = np.arange(T)
    for vis, ratio, K in ((O.TOKEN, 1, 5), (O.POOLED, 4, 8)):
        prob = _problem(S=T, T=T, H=H, D=D, K=K, vis=vis, ratio=ratio)
        c = _bf16_bits_of_ints(rng.integers(0, 3, size=(ratio, D))) if vis == O.POOLED else None
        a = O.topk_rows(prob, qb, kb, w, rows, pool_coef=c)
        b = O.topk_rows_docs(prob, qb, kb, w, rows, [0, T], pool_coef=c)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    bounds = [0, 13, 14, 27, 40]   # a one-token document; lengths not multiples of 4
    prob = _problem(S=T, T=T, H=H, D=D, K=5)
    idx, ln, _, _ = O.topk_rows_docs(prob, qb, kb, w, rows, bounds)
    keys = O.decode_bf16(kb)
    for t in rows:
        d = int(np.searchsorted(bounds, t, side="right")) - 1
        s = O.score_keys(O.decode_bf16(qb[t]), w[t].astype(np.float64), keys)
        s[: bounds[d]] = -np.inf
        s[t + 1:] = -np.inf
        n = min(5, t - bounds[d] + 1)
        top = np.argsort(-s, kind="stable")[:n]
        assert idx[t, : ln[t]].tolist() == sorted(top.tolist()), t
    prob = _problem(S=T, T=T, H=H, D=D, K=8, vis=O.POOLED, ratio=4)
    c = _bf16_bits_of_ints(rng.integers(0, 3, size=(4, D)))
    idx, ln, _, _ = O.topk_rows_docs(prob, qb, kb, w, rows, bounds, pool_coef=c)
    for t in rows:
        d = int(np.searchsorted(bounds, t, side="right")) - 1
        b = bounds[d]
        row = idx[t, : ln[t]]
        assert ((row >= b) & (row <= t)).all(), t
        nc = (t - b + 1) // 4
        tail = list(range(b + 4 * nc, t + 1))
        body = row[: len(row) - len(tail)]
        assert row[len(body):].tolist() == tail, t
        assert len(body) % 4 == 0 and all((body[i] - b) % 4 == 0 and
                                          body[i:i + 4].tolist() == list(range(body[i], body[i] + 4))
                                          for i in range(0, len(body), 4)), t


def pin_documents_compressed(O):
    """Compressed keys in a packed batch ("Module 06 — DSA & KPool", §3 and
    "Ship it": nothing of one document may reach another's selection): a
    document starts on a whole compressed key, and the query at global
    position g in the document starting at token b sees compressed key j iff
    j >= b / ratio and ratio*j + ratio - 1 <= g.  Checked by brute force: the
    full score row over every compressed key, every other key excluded, a
    stable sort; a batch of one document equals the plain compressed indexer;
    a query within ratio - 1 tokens of its document start selects nothing."""
    rng = np.random.default_rng(43)
    H, D, m, K = 3, 8, 4, 5
    n_tok = 64
    T = n_tok // m
    qb = _bf16_bits_of_ints(rng.integers(-3, 4, size=(n_tok, H, D)))
    kb = _bf16_bits_of_ints(rng.integers(-3, 4, size=(T, D)))
    w = rng.integers(-2, 3, size=(n_tok, H)).astype(np.float32)
    rows = np.arange(n_tok)
    prob = _problem(S=n_tok, T=T, H=H, D=D, K=K, vis=O.COMPRESSED, ratio=m)
    a = O.topk_rows(prob, qb, kb, w, rows)
    b = O.topk_rows_docs(prob, qb, kb, w, rows, [0, n_tok])
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    bounds = [0, 12, 16, 40, 64]   # documents of 12, 4, 24 and 24 tokens
    idx, ln, _, _ = O.topk_rows_docs(prob, qb, kb, w, rows, bounds)
    keys = O.decode_bf16(kb)
    for t in rows:
        d = int(np.searchsorted(bounds, t, side="right")) - 1
        start = bounds[d]
        s = O.score_keys(O.decode_bf16(qb[t]), w[t].astype(np.float64), keys)
        allowed = np.array([j * m >= start and m * j + m - 1 <= t for j in range(T)])
        s[~allowed] = -np.inf
        n = min(K, int(allowed.sum()))
        top = np.argsort(-s, kind="stable")[:n]
        assert idx[t, : ln[t]].tolist() == sorted(top.tolist()), t
        if t - start < m - 1:
            assert ln[t] == 0, t


def pin_padded_batch(O):
    """Padded batches ("Module 06 — DSA & KPool", §3 and "Ship it": the watch
    lengths 3, 4, 5, 7, 8, 9 checked with and without padding): every real
    row of a padded batch equals the plain indexer run on its sequence alone
    (sliced out, positions from 0), shifted by the sequence's first row;
    padding rows select nothing; with no padding the batch equals a packed
    batch whose documents start at multiples of the stride."""
    rng = np.random.default_rng(47)
    H, D, stride = 3, 8, 12
    lens = [3, 4, 5, 7, 8, 9]
    n = stride * len(lens)
    qb = _bf16_bits_of_ints(rng.integers(-3, 4, size=(n, H, D)))
    kb = _bf16_bits_of_ints(rng.integers(-3, 4, size=(n, D)))
    w = rng.integers(-2, 3, size=(n, H)).astype(np.float32)
    rows = np.arange(n)
    for vis, ratio, K in ((O.TOKEN, 1, 4), (O.COMPRESSED, 4, 2), (O.POOLED, 4, 4)):
        c = _bf16_bits_of_ints(rng.integers(0, 3, size=(ratio, D))) if vis == O.POOLED else None
        keys_all = kb if vis != O.COMPRESSED else kb[: n // ratio]
        prob = _problem(S=n, T=keys_all.shape[0], H=H, D=D, K=K, vis=vis, ratio=ratio)
        idx, ln, _, _ = O.topk_rows_padded(prob, qb, keys_all, w, rows, lens, stride, pool_coef=c)
        for b, L in enumerate(lens):
            r0 = b * stride
            assert (ln[r0 + L: r0 + stride] == 0).all() and (idx[r0 + L: r0 + stride] == -1).all(), (vis, b)
            if vis == O.COMPRESSED:
                kk, shift = kb[r0 // ratio: (r0 + L) // ratio], r0 // ratio
                if kk.shape[0] == 0:
                    assert (ln[r0: r0 + L] == 0).all()
                    continue
            else:
                kk, shift = kb[r0: r0 + L], r0
            one = _problem(S=L, T=kk.shape[0], H=H, D=D, K=K, vis=vis, ratio=ratio)
            ri, rl, _, _ = O.topk_rows(one, qb[r0: r0 + L], kk, w[r0: r0 + L], np.arange(L), pool_coef=c)
            for j in range(L):
                assert ln[r0 + j] == rl[j], (vis, b, j)
                assert idx[r0 + j, : ln[r0 + j]].tolist() == (ri[j, : rl[j]] + shift).tolist(), (vis, b, j)
        full = [stride] * len(lens)
        a = O.topk_rows_padded(prob, qb, keys_all, w, rows, full, stride, pool_coef=c)
        bnd = [stride * i for i in range(len(lens) + 1)]
        d = O.topk_rows_docs(prob, qb, keys_all, w, rows, bnd, pool_coef=c)
        assert np.array_equal(a[0], d[0]) and np.array_equal(a[1], d[1]), vis


def pin_fp8_scales(O):
    """An FP8 value means code * row scale: doubling every key scale doubles
    every score and leaves the selection unchanged; a per-(query, head) scale
    acts on that head exactly like its weight."""
    rng = np.random.default_rng(29)
    H, D, T, K = 3, 8, 64, 9
    codes_q = rng.integers(0, 0x7E, size=(1, H, D)).astype(np.uint8)  # finite codes
    codes_k = rng.integers(0, 0x7E, size=(T, D)).astype(np.uint8)
    codes_q[..., ::2] |= 0x80
    codes_k[::3] |= 0x80
    w = np.array([[0.5, -1.0, 2.0]], dtype=np.float32)
    prob = _problem(S=1, T=T, H=H, D=D, K=K, dtype="fp8", q_pos0=T - 1)
    one = np.ones(T, np.float32)
    qs = np.ones((1, H), np.float32)
    i1, l1, s1, _ = O.topk_rows(prob, codes_q, codes_k, w, [0], q_scale_rows=qs, k_scale=one)
    i2, l2, s2, _ = O.topk_rows(prob, codes_q, codes_k, w, [0], q_scale_rows=qs, k_scale=2 * one)
    assert np.array_equal(i1, i2) and np.allclose(s2[0, : l2[0]], 2 * s1[0, : l1[0]], rtol=1e-12)
    qs2 = np.array([[2.0, 1.0, 1.0]], np.float32)
    w2 = np.array([[0.25, -1.0, 2.0]], np.float32)
    i3, l3, s3, _ = O.topk_rows(prob, codes_q, codes_k, w2, [0], q_scale_rows=qs2, k_scale=one)
    assert np.array_equal(i1, i3) and np.allclose(s3[0, : l3[0]], s1[0, : l1[0]], rtol=1e-12)
    # and the decoded value equals the library's cast times the scale
    k64 = torch.from_numpy(codes_k.copy()).view(torch.float8_e4m3fn).double().numpy()
    q64 = torch.from_numpy(codes_q.copy()).view(torch.float8_e4m3fn).double().numpy()[0]
    s_lib = np.maximum(k64 @ q64.T, 0.0) @ w[0].astype(np.float64)
    top = np.argsort(-s_lib, kind="stable")[:K]
    assert i1[0, : l1[0]].tolist() == sorted(top.tolist())


def pin_witness(O):
    """Seed threshold ([DoSA] 核心方法, first step): the seed rule by hand
    (negative, invisible and repeated or out-of-order keys dropped; a pooled
    position names its pool); seeds equal to the row's own top-K give exactly
    its K-th score; any K or more distinct visible seeds give at most that
    (brute force over the full score row); K copies of one key are one seed."""
    assert O.witness_seed_keys([5, 3, 5, 7, -1, 10**9, 8], 100, 50, O.TOKEN, 1).tolist() == [5, 7, 8]
    assert O.witness_seed_keys([8, 9, 10, 11, 12, 13, 14], 13, 100, O.POOLED, 4).tolist() == [2]
    assert O.witness_seed_keys([0, 2, 3, 1], 13, 100, O.COMPRESSED, 4).tolist() == [0, 2]
    rng = np.random.default_rng(41)
    H, D, T, K = 3, 8, 60, 6
    qb = _bf16_bits_of_ints(rng.integers(-3, 4, size=(T, H, D)))
    kb = _bf16_bits_of_ints(rng.integers(-3, 4, size=(T, D)))
    w = rng.integers(-2, 3, size=(T, H)).astype(np.float32)
    rows = np.arange(T)
    prob = _problem(S=T, T=T, H=H, D=D, K=K)
    idx, ln, _, tau = O.topk_rows(prob, qb, kb, w, rows)
    got = O.witness_threshold(prob, qb, kb, w, rows, idx)
    full = ln == K
    assert np.array_equal(got[full], tau[full]) and np.isnan(got[~full]).all()
    keys = O.decode_bf16(kb)
    for t in range(K, T):
        s = np.sort(O.score_keys(O.decode_bf16(qb[t]), w[t].astype(np.float64), keys[: t + 1]))[::-1]
        for _ in range(3):
            n = int(rng.integers(K, t + 2))
            seeds = np.sort(rng.choice(t + 1, size=n, replace=False))
            sub = np.sort(O.score_keys(O.decode_bf16(qb[t]), w[t].astype(np.float64), keys[seeds]))[::-1]
            th = O.witness_threshold(prob, qb[t:t + 1], kb, w[t:t + 1], [t], seeds[None, :])[0]
            assert th == sub[K - 1] and th <= s[K - 1]
    best = int(np.argmax(O.score_keys(O.decode_bf16(qb[T - 1]), w[T - 1].astype(np.float64), keys)))
    assert np.isnan(O.witness_threshold(prob, qb[-1:], kb, w[-1:], [T - 1], np.full((1, K), best))[0])
    # pooled: the row's own output (token positions, then the tail) gives its K-th pool score
    c = _bf16_bits_of_ints(rng.integers(0, 3, size=(4, D)))
    pprob = _problem(S=T, T=T, H=H, D=D, K=8, vis=O.POOLED, ratio=4)
    pidx, pln, _, ptau = O.topk_rows(pprob, qb, kb, w, rows, pool_coef=c)
    pgot = O.witness_threshold(pprob, qb, kb, w, rows, pidx, pool_coef=c)
    pfull = ~np.isnan(ptau)
    assert pfull.any() and np.array_equal(pgot[pfull], ptau[pfull]) and np.isnan(pgot[~pfull]).all()
    # compressed keys and FP8 storage: the row's own output again gives its K-th score
    cprob = _problem(S=T, T=T // 4, H=H, D=D, K=4, vis=O.COMPRESSED, ratio=4)
    cidx, _, _, ctau = O.topk_rows(cprob, qb, kb[: T // 4], w, rows)
    cgot = O.witness_threshold(cprob, qb, kb[: T // 4], w, rows, cidx)
    cfull = ~np.isnan(ctau)
    assert cfull.any() and np.array_equal(cgot[cfull], ctau[cfull]) and np.isnan(cgot[~cfull]).all()
    codes_q = rng.integers(0, 0x7E, size=(4, H, D)).astype(np.uint8)
    codes_k = rng.integers(0, 0x7E, size=(T, D)).astype(np.uint8)
    codes_k[::2] |= 0x80
    qs = rng.uniform(0.5, 2.0, size=(4, H)).astype(np.float32)
    ks = rng.uniform(0.5, 2.0, size=T).astype(np.float32)
    fprob = _problem(S=4, T=T, H=H, D=D, K=K, dtype="fp8", q_pos0=T - 4)
    fidx, _, _, ftau = O.topk_rows(fprob, codes_q, codes_k, w[:4], np.arange(4), q_scale_rows=qs, k_scale=ks)
    fgot = O.witness_threshold(fprob, codes_q, codes_k, w[:4], np.arange(4), fidx, q_scale_rows=qs, k_scale=ks)
    # non-integer values: the two paths score different key subsets, so allow
    # a difference in the last bits of the FP64 sums
    assert np.allclose(fgot, ftau, rtol=1e-12, atol=0.0) and not np.isnan(fgot).any()


PINS = [
    pin_hand_worked,
    pin_integer_bruteforce,
    pin_score_properties,
    pin_selection_bruteforce,
    pin_selection_dominance,
    pin_chunked_equals_materialised,
    pin_row_invariants,
    pin_prefix_closed_form,
    pin_visibility_closed_forms,
    pin_watch_lengths,
    pin_slot_count,
    pin_pooled_keys,
    pin_pooled_keys_inexact_sums,
    pin_e4m3_decoder,
    pin_bf16_codec,
    pin_pair_overlap,
    pin_pair_regions,
    pin_documents,
    pin_documents_compressed,
    pin_padded_batch,
    pin_fp8_scales,
    pin_witness,
]
