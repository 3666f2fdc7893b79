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
C = sum_h |w_h| |d_h|.  The residual allowance may instead be the same page's
joint bound (技术新颖性): with x_h = w_h d_h,
  sum_h [x_h.k]_+ <= 1/2 (|sum_h x_h| + sqrt(sum_{h,l} |x_h.x_l|)) |k|,
and the CUDA path uses the smaller of the two.  This test restates both
constructions independently in NumPy and checks U >= s for every key, for
random and for correlated heads, and that the joint allowance is never larger.
"""

import numpy as np


def _certificate(q, w, r, joint=False):
    H, _ = q.shape
    nq = np.linalg.norm(q, axis=1)
    wt = w[:r].copy()
    C = 0.0
    xs = []
    for h in range(r, H):
        proj = q[:r] @ q[h] / np.maximum(nq[:r], 1e-300)
        j = int(np.argmax(proj))
        dot = float(q[h] @ q[j])
        beta = dot / nq[j] ** 2 if (dot > 0 and nq[j] > 0) else 0.0
        d = q[h] - beta * q[j]
        wt[j] += w[h] * beta
        C += abs(w[h]) * np.linalg.norm(d)
        xs.append(w[h] * d)
    if joint and xs:
        x = np.array(xs)
        e_joint = 0.5 * (np.linalg.norm(x.sum(axis=0)) + np.sqrt(np.abs(x @ x.T).sum()))
        assert e_joint <= C * (1 + 1e-12)
        C = min(C, e_joint)
    return wt, C


def _check(q, w, keys, r, joint=False):
    wt, C = _certificate(q, w, r, joint)
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


def test_joint_bound_holds_and_is_tighter():
    """The joint residual allowance bounds the score on random, correlated and
    anticorrelated heads with signed weights, and on random heads (nearly
    orthogonal residuals) it is far below the per-head sum."""
    rng = np.random.default_rng(3)
    for kind in ("random", "correlated", "anti"):
        for _ in range(10):
            H, D, n, r = 64, 128, 400, 16
            if kind == "random":
                q = rng.standard_normal((H, D))
            elif kind == "correlated":
                q = rng.standard_normal(D)[None, :] + 0.3 * rng.standard_normal((H, D))
            else:
                sign = np.where(rng.random(H) < 0.5, -1.0, 1.0)
                q = sign[:, None] * rng.standard_normal(D)[None, :] + 0.3 * rng.standard_normal((H, D))
            w = rng.standard_normal(H) / 8
            keys = rng.standard_normal((n, D)) * 2
            _check(q, w, keys, r, joint=True)
    q = rng.standard_normal((64, 128))
    w = rng.standard_normal(64) / 8
    assert _certificate(q, w, 16, joint=True)[1] < 0.5 * _certificate(q, w, 16)[1]


def test_joint_bound_is_attained_by_aligned_residuals():
    """Two residuals along the same direction and a key along it: the joint
    allowance equals the residual sum exactly (no slack to drop)."""
    u = np.zeros(8)
    u[0] = 1.0
    x = np.array([2.0 * u, 3.0 * u])
    k = u * 5.0
    r_sum = np.maximum(x @ k, 0.0).sum()
    e_joint = 0.5 * (np.linalg.norm(x.sum(axis=0)) + np.sqrt(np.abs(x @ x.T).sum()))
    assert abs(e_joint * np.linalg.norm(k) - r_sum) < 1e-12
