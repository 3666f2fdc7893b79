"""The pruning certificate's inequality, checked in float64 on the CPU.

"DoSA: Dots Sparse Attention", 核心方法 (core method): a key may be skipped
when an upper bound U_i of its score is below a lower bound of the K-th score.
The bound used by the CUDA path keeps r heads exactly and folds every other
head h onto an anchor j in the kept set with beta = [q_h.q_j]_+ / |q_j|^2 and
d_h = q_h - beta q_j:

  w_h > 0:  w_h [q_h.k]_+ <= w_h beta [q_j.k]_+ + w_h |d_h| |k|   (projection)
  w_h < 0:  w_h [q_h.k]_+ <= w_h beta [q_j.k]_+ + |w_h| |d_h| |k|  (the same
            projection read as a lower bound of [q_h.k]_+)

so U = sum_j w~_j [q_j.k]_+ + C |k|, w~_j = w_j + sum_{h -> j} w_h beta_h,
C = sum_h |w_h| |d_h|.  This test restates that construction independently
in NumPy and checks U >= s for every key, for random and for correlated heads.
"""

import numpy as np


def _certificate(q, w, r):
    H, _ = q.shape
    nq = np.linalg.norm(q, axis=1)
    wt = w[:r].copy()
    C = 0.0
    for h in range(r, H):
        proj = q[:r] @ q[h] / np.maximum(nq[:r], 1e-300)
        j = int(np.argmax(proj))
        dot = float(q[h] @ q[j])
        beta = dot / nq[j] ** 2 if (dot > 0 and nq[j] > 0) else 0.0
        d = np.linalg.norm(q[h] - beta * q[j])
        wt[j] += w[h] * beta
        C += abs(w[h]) * d
    return wt, C


def _check(q, w, keys, r):
    wt, C = _certificate(q, w, r)
    s = np.maximum(keys @ q.T, 0.0) @ w
    U = np.maximum(keys @ q[:r].T, 0.0) @ wt + C * np.linalg.norm(keys, axis=1)
    assert np.all(U >= s - 1e-9 * (1 + np.abs(s))), (U - s).min()
    return U, s


def test_bound_holds_on_random_heads():
    rng = np.random.default_rng(0)
    for _ in range(20):
        H, D, n, r = 64, 128, 500, 16
        q = rng.standard_normal((H, D))
        w = rng.standard_normal(H) / 8
        keys = rng.standard_normal((n, D))
        _check(q, w, keys, r)


def test_bound_holds_and_is_tight_on_correlated_heads():
    rng = np.random.default_rng(1)
    H, D, n, r = 64, 128, 2000, 16
    z = rng.standard_normal(D)
    q = z[None, :] + 0.01 * rng.standard_normal((H, D))
    w = np.abs(rng.standard_normal(H)) / 8
    keys = rng.standard_normal((n, D))
    U, s = _check(q, w, keys, r)
    # near-identical heads: the bound is close to the score for high-scoring keys
    top = np.argsort(-s)[:20]
    assert np.all(U[top] - s[top] <= 0.2 * s[top])


def test_bound_holds_with_signed_weights_and_anticorrelated_heads():
    rng = np.random.default_rng(2)
    H, D, n, r = 32, 64, 400, 16
    base = rng.standard_normal(D)
    sign = np.where(rng.random(H) < 0.5, -1.0, 1.0)
    q = sign[:, None] * base[None, :] + 0.3 * rng.standard_normal((H, D))
    w = rng.standard_normal(H)
    keys = rng.standard_normal((n, D)) * 3
    _check(q, w, keys, r)
