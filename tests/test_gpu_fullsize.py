"""The five workloads at full size, in the launch configuration bench.py times,
checked against the oracle on seeded samples of 1,024 query rows (the first
rows, rows around K and around pool boundaries, the last rows, the rest
uniform); the tiny exactness case on every row.  With HWR_PARITY_RECORD set to
a file name, each workload appends one JSON line of recall and score-error
figures to it."""

import json
import os

import numpy as np
import pytest
import torch

from head_weighted_relu_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu

# rows the FP64 oracle checks per workload (None: every row)
ROWS = {"tiny_int_512": None, "dsa_prefill_64k": 1024, "csa_m4_256k": 1024,
        "pooled_tail_128k": 1024, "long_1m_fp8": 1024}


def _threads():
    try:
        cores = len(os.sched_getaffinity(0))
    except Exception:
        cores = os.cpu_count() or 1
    return max(1, min(cores, 16))


@pytest.mark.parametrize("name", list(ROWS))
def test_full_size(cuda_ok, name):
    wl = W.WORKLOADS[name]
    inp = W.generate(wl, "cuda")
    gpu = parity.run_gpu(wl, inp)
    n = ROWS[name]
    rows = np.arange(wl.S) if n is None else W.sample_rows(wl, n)
    ref = parity.oracle_rows(wl, inp, rows, threads=_threads())
    stats = {"workload": name, "sampled_rows": int(len(rows))}
    if wl.values == "int":
        parity.assert_exact(gpu, ref, rows)
        stats.update(exact=True, mean_recall=1.0, min_recall=1.0)
    else:
        recall = parity.assert_tolerant(wl, gpu, ref, rows, stats=stats)
        print(f"{name}: mean recall {recall:.6f} over {len(rows)} rows")
    rec = os.environ.get("HWR_PARITY_RECORD")
    if rec:
        with open(rec, "a") as f:
            f.write(json.dumps(stats) + "\n")
    # properties that hold on every row, checked on all of them
    idx, ln = gpu[0], gpu[1]
    valid = torch.arange(idx.shape[1], device=idx.device)[None, :] < ln[:, None]
    assert bool(((idx >= 0) == valid).all()), "padding must be -1 exactly after the valid length"
    d = idx[:, 1:] - idx[:, :-1]
    both = valid[:, 1:]
    assert bool((d[both] > 0).all()), "valid prefixes must be strictly ascending"
