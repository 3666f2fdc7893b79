"""The five workloads at full size, in the launch configuration bench.py times,
checked against the oracle on seeded samples of query rows (the first rows,
rows around K and around pool boundaries, the last row, the rest uniform)."""

import numpy as np
import pytest
import torch

from head_weighted_relu_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu

# rows the FP64 oracle checks per workload (the 1M-key rows cost ~0.2 s each)
ROWS = {"tiny_int_512": None, "dsa_prefill_64k": 1024, "csa_m4_256k": 1024,
        "pooled_tail_128k": 1024, "long_1m_fp8": 128}


@pytest.mark.parametrize("name", list(ROWS))
def test_full_size(cuda_ok, name):
    wl = W.WORKLOADS[name]
    inp = W.generate(wl, "cuda")
    gpu = parity.run_gpu(wl, inp)
    n = ROWS[name]
    rows = np.arange(wl.S) if n is None else W.sample_rows(wl, n)
    ref = parity.oracle_rows(wl, inp, rows)
    if wl.values == "int":
        parity.assert_exact(gpu, ref, rows)
    else:
        recall = parity.assert_tolerant(wl, gpu, ref, rows)
        print(f"{name}: mean recall {recall:.6f} over {len(rows)} rows")
    # properties that hold on every row, checked on all of them
    idx, ln = gpu[0], gpu[1]
    valid = torch.arange(idx.shape[1], device=idx.device)[None, :] < ln[:, None]
    assert bool(((idx >= 0) == valid).all()), "padding must be -1 exactly after the valid length"
    d = idx[:, 1:] - idx[:, :-1]
    both = valid[:, 1:]
    assert bool((d[both] > 0).all()), "valid prefixes must be strictly ascending"
