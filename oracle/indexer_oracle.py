"""Oracle for the DSA lightning indexer: head-weighted ReLU scores, exact top-K.

TEST INFRASTRUCTURE ONLY (see the package docstring): plain NumPy in IEEE
binary64, one query row at a time, a full score row per query followed by a
stable sort.  Library primitives used as single steps: a matrix product
(numpy.matmul) and a stable sort (numpy.argsort, kind="stable").

Sources, cited by page title and section:
  [DoSA]   "DoSA: Dots Sparse Attention" (paper summary), section 前置知识
           (background): the indexer scores every visible key with
           s_i = sum_h w_h [q_h . k_i]_+, ReLU [.]_+, head weights of either
           sign; section 研究动机 (motivation): the result is the exact top-K
           under one fixed tie rule.
  [KPool]  "Module 06 — DSA & KPool: Selective Retrieval", §2 (the selection
           budget: 2,048 positions = 512 pools of 4; selected pools expand to
           their tokens; the still-incomplete pool is appended as a tail of at
           most 3 positions; 2,051 slots) and §3 (a pool becomes selectable once
           its final token is causally visible; position i sees j iff j <= i).
  [Overlap] "Adjacent-Query KV-Index Overlap in 256K DSA Training", §1 (pairs
           (q0,q1),(q2,q3),...; valid top-k length) and §3 (indices sorted by KV
           index; exact intersection sizes).
  [StreamIndex] arXiv 2605.02568, abstract: compressed (CSA) keys with ratio
           m = 4; the materialised score row is the ground truth.

Readings taken where the pages are silent or garbled:
  * the weights are per query: w[t, h];
  * selection order: higher score first, then lower key index; -0.0 == +0.0;
  * a row with fewer visible keys than the budget selects all of them;
  * compressed key j stands for tokens m*j .. m*j+m-1 and is visible to the
    query at global position g iff its last token m*j+m-1 <= g (the pool
    completion rule of [KPool] §3 applied to compressed blocks);
  * pooled key p = RNE_bf16(exact sum_j c[j] (*) k[m*p+j]) (channel-wise
    weighted representation of a complete pool, [KPool] §2), rounded once;
  * the tail of the query's own incomplete pool is appended after the expanded
    pools;
  * an FP8 e4m3 value is multiplied by its FP32 row scale.
"""

from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

TOKEN, COMPRESSED, POOLED = 0, 1, 2


# ----------------------------------------------------------------------------
# Storage formats (decoded from their definitions, not through a library cast)
# ----------------------------------------------------------------------------

def decode_bf16(bits) -> np.ndarray:
    """bfloat16 bit patterns -> float64.

    bfloat16 is the upper half of an IEEE binary32 word, so widening the bits
    by 16 zero bits gives the binary32 value exactly, and binary32 -> binary64
    is exact.
    """
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def _e4m3_table() -> np.ndarray:
    """All 256 FP8 e4m3 values, from the format's definition.

    1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent field 0
    encodes subnormals man/8 * 2^(1-7); the pattern S.1111.111 is NaN; there
    is no infinity, so the largest finite value is 1.75 * 2^8 = 448.
    """
    t = np.empty(256, dtype=np.float64)
    for byte in range(256):
        sign = -1.0 if byte & 0x80 else 1.0
        e = (byte >> 3) & 0xF
        m = byte & 0x7
        if e == 0xF and m == 0x7:
            t[byte] = math.nan
        elif e == 0:
            t[byte] = sign * (m / 8.0) * 2.0 ** (1 - 7)
        else:
            t[byte] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return t


_E4M3 = _e4m3_table()


def decode_e4m3(codes) -> np.ndarray:
    """FP8 e4m3 codes (uint8) -> float64 through the definition table."""
    return _E4M3[np.asarray(codes).astype(np.uint8)]


def round_to_bf16_bits(x) -> np.ndarray:
    """Round binary64 values to bfloat16 (round to nearest, ties to even).

    bfloat16 keeps 8 significant bits and binary32's exponent range.  A normal
    value x = f * 2^e with 0.5 <= |f| < 1 becomes rint(f * 2^8) * 2^(e-8);
    numpy.rint rounds half to even and f * 2^8 is exact.  Below 2^-126 the
    spacing is fixed at 2^-133 (subnormals).  Results of magnitude 2^128 or
    more overflow to infinity.  The rounded value has at most 8 significant
    bits, so it converts to binary32 exactly and its upper 16 bits are the
    bfloat16 pattern.
    """
    x = np.asarray(x, dtype=np.float64)
    f, e = np.frexp(x)
    y = np.ldexp(np.rint(np.ldexp(f, 8)), e - 8)
    small = np.abs(x) < 2.0 ** -126
    y = np.where(small, np.ldexp(np.rint(np.ldexp(x, 133)), -133), y)
    y = np.where(np.abs(y) >= 2.0 ** 128, np.copysign(np.inf, x), y)
    with np.errstate(invalid="ignore"):
        bits = (y.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    bits = np.where(np.isnan(x), np.uint16(0x7FC0), bits)
    return bits.astype(np.uint16)


def _round_fraction_to_bf16_bits(v: Fraction) -> int:
    """Exact rational -> bfloat16 (RNE); used only where a float sum was inexact."""
    if v == 0:
        return 0
    sign = 0x8000 if v < 0 else 0
    a = abs(v)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    # correct the floating estimate of floor(log2(a))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    quantum = Fraction(2) ** (max(e, -126) - 7)
    r = a / quantum
    n = r.numerator // r.denominator
    rem = r - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    y = float(n * quantum)
    if y >= 2.0 ** 128:
        return sign | 0x7F80
    return sign | int(np.array([y], dtype=np.float32).view(np.uint32)[0] >> 16)


# ----------------------------------------------------------------------------
# Visibility ([KPool] §3; [StreamIndex] abstract for compressed keys)
# ----------------------------------------------------------------------------

def visible_keys(g: int, n_keys: int, visibility: int, ratio: int) -> np.ndarray:
    """Indices of the keys visible to the query at global position g, ascending.

    TOKEN: token key i is visible iff i <= g (a position sees itself).
    COMPRESSED / POOLED: key j summarises tokens ratio*j .. ratio*j+ratio-1 and
    becomes visible only once its final token is visible: ratio*j+ratio-1 <= g.
    """
    j = np.arange(n_keys, dtype=np.int64)
    if visibility == TOKEN:
        mask = j <= g
    elif visibility in (COMPRESSED, POOLED):
        mask = ratio * j + ratio - 1 <= g
    else:
        raise ValueError(f"unknown visibility {visibility}")
    return j[mask]


def incomplete_tail(g: int, ratio: int) -> np.ndarray:
    """Positions of the query's own pool that are visible while that pool is
    still incomplete ([KPool] §2): the pool holding g is p = g // ratio; if g
    is not its final token, its positions ratio*p .. g form the tail."""
    p = g // ratio
    last = ratio * p + ratio - 1
    if last <= g:
        return np.zeros(0, dtype=np.int64)
    return np.arange(ratio * p, g + 1, dtype=np.int64)


# ----------------------------------------------------------------------------
# Pooled keys ([KPool] §2: channel-wise weighted representation of a pool)
# ----------------------------------------------------------------------------

def _two_sum(a: np.ndarray, b: np.ndarray):
    """Knuth's error-free transformation: a + b = s + err exactly."""
    s = a + b
    bb = s - a
    err = (a - (s - bb)) + (b - bb)
    return s, err


def pooled_keys(k_bits, c_bits, ratio: int) -> np.ndarray:
    """bfloat16 bits of kp[p, d] = RNE_bf16( sum_j c[j, d] * k[ratio*p + j, d] ).

    Products of two bfloat16 values are exact in binary64.  The sum is taken
    in binary64 left to right, and Knuth's TwoSum checks that every addition
    was exact; any element where one was not is recomputed with exact
    rationals.  The exact sum is then rounded once to bfloat16.
    """
    k = decode_bf16(k_bits)
    c = decode_bf16(c_bits)
    n_pools = k.shape[0] // ratio
    d = k.shape[1]
    kk = k[: n_pools * ratio].reshape(n_pools, ratio, d)
    prods = kk * c[None, :, :]
    acc = prods[:, 0, :].copy()
    inexact = np.zeros(acc.shape, dtype=bool)
    for j in range(1, ratio):
        acc, err = _two_sum(acc, prods[:, j, :])
        inexact |= err != 0
    out = round_to_bf16_bits(acc)
    for p, dd in zip(*np.nonzero(inexact)):
        exact = sum(Fraction(float(kk[p, j, dd])) * Fraction(float(c[j, dd])) for j in range(ratio))
        out[p, dd] = _round_fraction_to_bf16_bits(exact)
    return out


# ----------------------------------------------------------------------------
# Score ([DoSA] 前置知识) and selection ([DoSA] 研究动机; [Overlap] §3)
# ----------------------------------------------------------------------------

def score_keys(q_t: np.ndarray, w_t: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """s_i = sum_h w[h] * max(0, q[h] . k_i) for each row k_i of `keys`.

    q_t: [H, D] float64, w_t: [H] float64 (signed), keys: [n, D] float64.
    -0.0 is replaced by +0.0 (x + 0.0 does that under round-to-nearest).
    """
    dots = keys @ q_t.T                  # [n, H]: q_h . k_i
    relu = np.maximum(dots, 0.0)         # [q_h . k_i]_+
    s = relu @ w_t                       # sum over heads with signed weights
    return s + 0.0


def select_topk(s: np.ndarray, keys: np.ndarray, ksel: int):
    """Exact top-ksel of (score, key) pairs, returned sorted by key index.

    The order is: higher score first, then lower key index.  `keys` is
    ascending, so a stable sort on descending score keeps the lower index first
    among equal scores.  Rows with fewer than ksel keys select all of them.

    Returns (selected keys ascending, their scores, tau) where tau is the
    ksel-th best score (NaN when the row has fewer than ksel keys).
    """
    n = s.shape[0]
    order = np.argsort(-s, kind="stable")
    take = order[: min(ksel, n)]
    tau = float(s[order[ksel - 1]]) if n >= ksel else math.nan
    by_key = take[np.argsort(keys[take], kind="stable")]
    return keys[by_key], s[by_key], tau


def out_width(K: int, visibility: int, ratio: int) -> int:
    """Row width of the index output: the budget, plus ratio-1 tail slots for
    pooled selection ([KPool] §2: 512 pools * 4 + 3 = 2,051)."""
    return K + ratio - 1 if visibility == POOLED else K


def _decode_keys(problem: dict, k, k_scale, pool_coef):
    if problem["visibility"] == POOLED:
        kp = pooled_keys(k, pool_coef, problem["ratio"])
        return decode_bf16(kp)
    if problem["dtype"] == "fp8":
        return decode_e4m3(k) * np.asarray(k_scale, dtype=np.float64)[:, None]
    return decode_bf16(k)


def topk_rows(problem: dict, q_rows, k, w_rows, rows, q_scale_rows=None,
              k_scale=None, pool_coef=None, keys_f64=None):
    """Indexer output for the query rows `rows`.

    problem: dict with S, T, H, D, q_pos0, visibility, ratio, K, dtype
             ("bf16" or "fp8").  T counts token keys (TOKEN, POOLED) or
             compressed keys (COMPRESSED).
    q_rows:  [R, H, D] storage (bf16 bit patterns or e4m3 codes) of the rows.
    k:       [T, D] storage of all keys.
    w_rows:  [R, H] float32 weights of the rows.
    rows:    [R] query row numbers t; the global position is q_pos0 + t.
    q_scale_rows [R, H], k_scale [T]: FP32 row scales for FP8 storage.
    pool_coef: [ratio, D] bfloat16 bits of the pooling coefficients.
    keys_f64: optional pre-decoded keys (as returned by decode_keys_for).

    Returns (idx [R, W] int32 padded with -1, len [R] int32,
             score [R, W] float64 (NaN for tail and padding), tau [R]).
    """
    vis_mode = problem["visibility"]
    ratio = int(problem["ratio"]) if vis_mode != TOKEN else 1
    K = int(problem["K"])
    width = out_width(K, vis_mode, ratio)
    if keys_f64 is None:
        keys_f64 = _decode_keys(problem, k, k_scale, pool_coef)
    n_keys = keys_f64.shape[0]
    ksel = K // ratio if vis_mode == POOLED else K
    R = len(rows)
    out_idx = np.full((R, width), -1, dtype=np.int32)
    out_len = np.zeros(R, dtype=np.int32)
    out_score = np.full((R, width), math.nan, dtype=np.float64)
    taus = np.full(R, math.nan, dtype=np.float64)
    for r in range(R):
        g = int(problem["q_pos0"]) + int(rows[r])
        vis = visible_keys(g, n_keys, vis_mode, ratio)
        if problem["dtype"] == "fp8":
            q_t = decode_e4m3(q_rows[r]) * np.asarray(q_scale_rows[r], dtype=np.float64)[:, None]
        else:
            q_t = decode_bf16(q_rows[r])
        w_t = np.asarray(w_rows[r], dtype=np.float64)
        if vis.size and vis[-1] == vis.size - 1:
            block = keys_f64[: vis.size]          # a prefix: a view, no copy
        else:
            block = keys_f64[vis]
        s = score_keys(q_t, w_t, block)
        sel, ssel, tau = select_topk(s, vis, ksel)
        taus[r] = tau
        if vis_mode == POOLED:
            pos = (sel[:, None] * ratio + np.arange(ratio)[None, :]).reshape(-1)
            sc = np.repeat(ssel, ratio)
            tail = incomplete_tail(g, ratio)
            pos = np.concatenate([pos, tail])
            sc = np.concatenate([sc, np.full(tail.size, math.nan)])
        else:
            pos, sc = sel, ssel
        n = pos.size
        out_idx[r, :n] = pos
        out_len[r] = n
        out_score[r, :n] = sc
    return out_idx, out_len, out_score, taus


def witness_seed_keys(seed_row, g: int, n_keys: int, visibility: int, ratio: int) -> np.ndarray:
    """The distinct visible key rows that one row of seeds names, in order.

    [DoSA] 核心方法 (first step) scores a set of at least K visible seed keys
    exactly; a key counted twice would make its K-th score too high, so each
    key counts once.  An entry e names key row e (for POOLED a token position,
    which names the pool e // ratio holding it).  An entry is dropped when it
    is negative, when the key it names is not visible at g, or when that key is
    at or below the largest key kept so far (rows in ascending order are used
    whole).
    """
    n_vis = visible_keys(g, n_keys, visibility, ratio).size   # the visible keys are 0 .. n_vis-1
    kept = []
    top = -1
    for e in np.asarray(seed_row).tolist():
        if e < 0:
            continue
        r = e // ratio if visibility == POOLED else e
        if r >= n_vis or r <= top:
            continue
        kept.append(r)
        top = r
    return np.asarray(kept, dtype=np.int64)


def witness_threshold(problem: dict, q_rows, k, w_rows, rows, seeds, q_scale_rows=None,
                      k_scale=None, pool_coef=None, keys_f64=None) -> np.ndarray:
    """tau[r]: the K-th largest exact score over the distinct visible seeds of
    query row rows[r] ([DoSA] 核心方法, first step: a lower bound of the row's
    K-th score, since those seeds are some of its visible keys), NaN when the
    row has fewer than K (K / ratio pools for POOLED) such seeds.
    Arguments as topk_rows, plus seeds [R, n] (one row of seeds per query row).
    """
    vis_mode = problem["visibility"]
    ratio = int(problem["ratio"]) if vis_mode != TOKEN else 1
    K = int(problem["K"])
    ksel = K // ratio if vis_mode == POOLED else K
    if keys_f64 is None:
        keys_f64 = _decode_keys(problem, k, k_scale, pool_coef)
    taus = np.full(len(rows), math.nan, dtype=np.float64)
    for r in range(len(rows)):
        g = int(problem["q_pos0"]) + int(rows[r])
        sk = witness_seed_keys(seeds[r], g, keys_f64.shape[0], vis_mode, ratio)
        if sk.size < ksel:
            continue
        if problem["dtype"] == "fp8":
            q_t = decode_e4m3(q_rows[r]) * np.asarray(q_scale_rows[r], dtype=np.float64)[:, None]
        else:
            q_t = decode_bf16(q_rows[r])
        s = score_keys(q_t, np.asarray(w_rows[r], dtype=np.float64), keys_f64[sk])
        taus[r] = float(np.sort(s)[::-1][ksel - 1])
    return taus


def topk_rows_docs(problem: dict, q_rows, k, w_rows, rows, doc_bounds, q_scale_rows=None,
                   k_scale=None, pool_coef=None):
    """Indexer output for query rows of a packed batch of documents.

    Token positions [doc_bounds[d], doc_bounds[d+1]) form document d; a query
    sees only its own document, and pools never cross a document boundary
    ("Module 06 — DSA & KPool: Selective Retrieval", §3 and "Ship it": in a
    packed-document batch no pool may span a document boundary, and no token
    of one document may reach another document's selection).  For the query at global
    position g in document d starting at token b:
      TOKEN       keys b .. g;
      COMPRESSED  compressed keys j with j >= b / ratio and ratio*j+ratio-1 <= g
                  (documents start on a multiple of the ratio);
      POOLED      the document's pools: pool p covers tokens b+ratio*p ..
                  b+ratio*p+ratio-1, its key pooled from those tokens, visible
                  once complete; selected pools expand to their tokens, then
                  the tokens b+ratio*nc .. g of the document's incomplete pool.
    Indices are global token (or compressed-key) positions.  Arguments and
    results as topk_rows.
    """
    vis_mode = problem["visibility"]
    ratio = int(problem["ratio"]) if vis_mode != TOKEN else 1
    K = int(problem["K"])
    width = out_width(K, vis_mode, ratio)
    ksel = K // ratio if vis_mode == POOLED else K
    bounds = np.asarray(doc_bounds, dtype=np.int64)
    R = len(rows)
    out_idx = np.full((R, width), -1, dtype=np.int32)
    out_len = np.zeros(R, dtype=np.int32)
    out_score = np.full((R, width), math.nan, dtype=np.float64)
    taus = np.full(R, math.nan, dtype=np.float64)
    if vis_mode == POOLED:
        tokens = None
    else:
        tokens = _decode_keys(problem, k, k_scale, pool_coef)
    pooled_cache = {}
    for r in range(R):
        g = int(problem["q_pos0"]) + int(rows[r])
        d = int(np.searchsorted(bounds, g, side="right")) - 1
        b = int(bounds[d])
        if problem["dtype"] == "fp8":
            q_t = decode_e4m3(q_rows[r]) * np.asarray(q_scale_rows[r], dtype=np.float64)[:, None]
        else:
            q_t = decode_bf16(q_rows[r])
        w_t = np.asarray(w_rows[r], dtype=np.float64)
        if vis_mode == TOKEN:
            vis = np.arange(b, g + 1, dtype=np.int64)
            block = tokens[vis]
        elif vis_mode == COMPRESSED:
            j = np.arange(tokens.shape[0], dtype=np.int64)
            vis = j[(j >= b // ratio) & (ratio * j + ratio - 1 <= g)]
            block = tokens[vis]
        else:
            end = int(bounds[d + 1])
            if d not in pooled_cache:
                pooled_cache[d] = decode_bf16(pooled_keys(np.asarray(k)[b:end], pool_coef, ratio))
            doc_pools = pooled_cache[d]
            n_done = (g - b + 1) // ratio            # complete pools of the document
            vis = np.arange(n_done, dtype=np.int64)  # document-local pool numbers
            block = doc_pools[:n_done]
        s = score_keys(q_t, w_t, block)
        sel, ssel, tau = select_topk(s, vis, ksel)
        taus[r] = tau
        if vis_mode == POOLED:
            pos = (b + sel[:, None] * ratio + np.arange(ratio)[None, :]).reshape(-1)
            sc = np.repeat(ssel, ratio)
            doc_tail = np.arange(b + ratio * n_done, g + 1, dtype=np.int64)
            pos = np.concatenate((pos, doc_tail))
            sc = np.concatenate((sc, np.full(doc_tail.size, math.nan)))
        else:
            pos, sc = sel, ssel
        n = pos.size
        out_idx[r, :n] = pos
        out_len[r] = n
        out_score[r, :n] = sc
    return out_idx, out_len, out_score, taus


def topk_rows_padded(problem: dict, q_rows, k, w_rows, rows, seq_lens, stride: int,
                     q_scale_rows=None, k_scale=None, pool_coef=None):
    """Indexer output for query rows of a padded batch.

    The batch holds len(seq_lens) sequences, each padded to `stride` token
    rows: sequence b occupies rows b*stride .. b*stride + seq_lens[b] - 1 of
    the queries and of the token keys, and the rest of its stride is padding.
    A padding position is never visible and a padding query row selects
    nothing (length 0, all -1).  Inside a sequence everything is as for one
    sequence of its own ("Module 06 — DSA & KPool: Selective Retrieval", §3
    and "Ship it": every watch length checked with and without padding), with
    positions relative to the sequence start: the query at position j of
    sequence b sees
      TOKEN       token keys b*stride .. b*stride + j;
      COMPRESSED  compressed keys b*stride/ratio + c with ratio*c+ratio-1 <= j
                  (stride a multiple of the ratio);
      POOLED      the sequence's pools, pool c formed from tokens
                  b*stride + ratio*c .. + ratio-1, visible once complete, then
                  the tail b*stride + ratio*nc .. b*stride + j.
    Indices are rows of the padded key array.  Arguments and results as
    topk_rows (problem["S"] = number of query rows of the padded batch).
    """
    vis_mode = problem["visibility"]
    ratio = int(problem["ratio"]) if vis_mode != TOKEN else 1
    K = int(problem["K"])
    width = out_width(K, vis_mode, ratio)
    ksel = K // ratio if vis_mode == POOLED else K
    R = len(rows)
    out_idx = np.full((R, width), -1, dtype=np.int32)
    out_len = np.zeros(R, dtype=np.int32)
    out_score = np.full((R, width), math.nan, dtype=np.float64)
    taus = np.full(R, math.nan, dtype=np.float64)
    tokens = None if vis_mode == POOLED else _decode_keys(problem, k, k_scale, pool_coef)
    pooled_cache = {}
    for r in range(R):
        t = int(rows[r])
        b, j = divmod(t, stride)
        if j >= int(seq_lens[b]):
            continue                                  # a padding query row
        start = b * stride
        if problem["dtype"] == "fp8":
            q_t = decode_e4m3(q_rows[r]) * np.asarray(q_scale_rows[r], dtype=np.float64)[:, None]
        else:
            q_t = decode_bf16(q_rows[r])
        w_t = np.asarray(w_rows[r], dtype=np.float64)
        if vis_mode == TOKEN:
            vis = np.arange(start, start + j + 1, dtype=np.int64)
            block = tokens[vis]
        elif vis_mode == COMPRESSED:
            c = np.arange((j + 1) // ratio, dtype=np.int64)      # complete compressed keys so far
            vis = start // ratio + c
            block = tokens[vis]
        else:
            if b not in pooled_cache:
                n_tok = int(seq_lens[b])
                pooled_cache[b] = decode_bf16(pooled_keys(np.asarray(k)[start:start + n_tok], pool_coef, ratio))
            n_done = (j + 1) // ratio
            vis = np.arange(n_done, dtype=np.int64)              # sequence-local pool numbers
            block = pooled_cache[b][:n_done]
        s = score_keys(q_t, w_t, block)
        sel, ssel, tau = select_topk(s, vis, ksel)
        taus[r] = tau
        if vis_mode == POOLED:
            pos = (start + sel[:, None] * ratio + np.arange(ratio)[None, :]).reshape(-1)
            sc = np.repeat(ssel, ratio)
            tail = np.arange(start + ratio * n_done, start + j + 1, dtype=np.int64)
            pos = np.concatenate((pos, tail))
            sc = np.concatenate((sc, np.full(tail.size, math.nan)))
        else:
            pos, sc = sel, ssel
        n = pos.size
        out_idx[r, :n] = pos
        out_len[r] = n
        out_score[r, :n] = sc
    return out_idx, out_len, out_score, taus


def decode_keys_for(problem: dict, k, k_scale=None, pool_coef=None) -> np.ndarray:
    """Decoded float64 keys (pooled keys for POOLED) for reuse across calls."""
    return _decode_keys(problem, k, k_scale, pool_coef)


# ----------------------------------------------------------------------------
# Adjacent-pair overlap ([Overlap] §1 and §3)
# ----------------------------------------------------------------------------

def pair_shared_counts(idx, lens) -> np.ndarray:
    """|A_{2p} ∩ A_{2p+1}| for the non-overlapping pairs (q0,q1), (q2,q3), ...

    Each row's valid prefix idx[r, :lens[r]] holds distinct indices.  The two
    prefixes are concatenated and sorted; every index present in both appears
    exactly twice, as two neighbours, so the count is the number of equal
    neighbours.  (A different method from the binary search of [Overlap] §3.)
    """
    idx = np.asarray(idx)
    lens = np.asarray(lens)
    n_pairs = idx.shape[0] // 2
    out = np.zeros(n_pairs, dtype=np.int32)
    for p in range(n_pairs):
        a = idx[2 * p, : lens[2 * p]]
        b = idx[2 * p + 1, : lens[2 * p + 1]]
        both = np.sort(np.concatenate([a, b]), kind="stable")
        out[p] = int(np.count_nonzero(both[1:] == both[:-1]))
    return out


def pair_regions(idx, lens, width: int):
    """The three index regions of each non-overlapping adjacent query pair.

    "Adjacent-Query KV-Index Overlap in 256K DSA Training", §6.1: a two-query
    cluster splits its selection into the indices both queries select, those
    only the left query (row 2p) selects, and those only the right query (row
    2p+1) selects; §6.4: each region goes to a buffer of fixed capacity (the
    row width), with its length as a device-side count.  Here the regions are
    the set intersection and the two set differences of the valid prefixes,
    each listed in ascending KV order and padded with -1.

    Returns shared, left, right [S/2, width] int32 and counts [S/2, 3] int32
    (shared, left-only, right-only).
    """
    idx = np.asarray(idx)
    lens = np.asarray(lens)
    n_pairs = idx.shape[0] // 2
    regions = [np.full((n_pairs, width), -1, dtype=np.int32) for _ in range(3)]
    counts = np.zeros((n_pairs, 3), dtype=np.int32)
    for p in range(n_pairs):
        a = set(int(v) for v in idx[2 * p, : lens[2 * p]])
        b = set(int(v) for v in idx[2 * p + 1, : lens[2 * p + 1]])
        for r, members in enumerate((a & b, a - b, b - a)):
            ordered = sorted(members)
            regions[r][p, : len(ordered)] = ordered
            counts[p, r] = len(ordered)
    return regions[0], regions[1], regions[2], counts

