"""Pool formation on the GPU (indexer_pool_keys, "Module 06 — DSA & KPool",
§2) bit-exact against the oracle where the binary64 running sum of a pool's
products is not exact: the hand-worked columns of
tests/golden/pooled_rounding_cases.txt and random columns whose products span
up to 2^80 in magnitude, plus signed zeros."""

import numpy as np
import pytest
import torch

import oracle
from tests import oracle_pins as P

pytestmark = pytest.mark.gpu


def _pool_on_gpu(k_bits, c_bits, ratio):
    from head_weighted_relu_b200 import indexer as I
    k = torch.from_numpy(k_bits.view(np.int16).copy()).view(torch.bfloat16).cuda()
    c = torch.from_numpy(c_bits.view(np.int16).copy()).view(torch.bfloat16).cuda()
    out = I.pool_keys(k, c, ratio)
    torch.cuda.synchronize()
    return out.cpu().view(torch.int16).numpy().view(np.uint16)


def test_pool_keys_hand_worked_columns(cuda_ok):
    cases = P.pooled_rounding_cases()
    D = len(cases)
    k = np.zeros((4, D), dtype=np.uint16)
    c = np.zeros((4, D), dtype=np.uint16)
    for d, (kv, cv, _) in enumerate(cases):
        k[:, d] = P._bf16_bits_of_fractions(kv)
        c[:, d] = P._bf16_bits_of_fractions(cv)
    got = _pool_on_gpu(k, c, 4)
    want = np.array([[w for _, _, w in cases]], dtype=np.uint16)
    assert np.array_equal(got, want), [(d, hex(int(a)), hex(int(b))) for d, (a, b) in
                                       enumerate(zip(got[0], want[0])) if a != b]
    assert np.array_equal(got, oracle.pooled_keys(k, c, 4))


@pytest.mark.parametrize("ratio", [4, 7])
def test_pool_keys_wide_exponents(cuda_ok, ratio):
    rng = np.random.default_rng(100 + ratio)
    n_pools, D = 512, 128
    mant = rng.integers(1, 256, size=(n_pools * ratio, D)) * rng.choice([-1, 1], size=(n_pools * ratio, D))
    expo = rng.integers(-40, 41, size=(n_pools * ratio, D))
    kf = torch.from_numpy(np.ldexp(mant.astype(np.float64), expo))
    cm = rng.integers(1, 256, size=(ratio, D)) * rng.choice([-1, 1], size=(ratio, D))
    cf = torch.from_numpy(np.ldexp(cm.astype(np.float64), rng.integers(-40, 41, size=(ratio, D))))
    k = kf.to(torch.bfloat16)
    c = cf.to(torch.bfloat16)
    assert torch.equal(k.double(), kf) and torch.equal(c.double(), cf)   # exact bf16 values
    k_bits = k.view(torch.int16).numpy().view(np.uint16)
    c_bits = c.view(torch.int16).numpy().view(np.uint16)
    # signed zeros: a column of -0 constituents, and one of +0 and -0 mixed
    k_bits[: ratio, 0] = 0x8000
    c_bits[:, 0] = 0x3F80
    k_bits[: ratio, 1] = [0x8000 if j % 2 else 0 for j in range(ratio)]
    got = _pool_on_gpu(k_bits, c_bits, ratio)
    want = oracle.pooled_keys(k_bits, c_bits, ratio)
    assert got[0, 0] == 0x8000 and want[0, 0] == 0x8000
    bad = np.argwhere(got != want)
    assert bad.size == 0, [(int(p), int(d), hex(int(got[p, d])), hex(int(want[p, d]))) for p, d in bad[:8]]
