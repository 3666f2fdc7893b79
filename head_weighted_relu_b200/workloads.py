"""Seeded synthetic inputs for the indexer, shaped like the source pages' workloads.

This module only draws random tensors and fixes shapes; it holds none of the
indexer's arithmetic (no scores, masks, pooling or selection), so both the CUDA
path and the CPU oracle can be fed from it.  Every draw is rounded to its
storage type here, once.

Workloads (names carry their sizes):
  tiny_int_512      S=T=512, H=4, D=64, K=64, token causal; integer q, k in
                    [-3, 3] and w in {-2..2}: every score is an exact integer.
  dsa_prefill_64k   S=T=65,536, H=64, D=128, K=2,048, token causal, N(0,1)
                    bf16 q, k; w ~ N(0, 1/H) fp32 (DSA prefill).
  dsa_prefill_16k   the same at S=T=16,384 (a profiling-sized case).
  csa_m4_256k       S=262,144 queries over T=65,536 compressed keys (m=4),
                    H=64, D=128, K=2,048 (V4-Flash-like CSA indexer shape).
  pooled_tail_128k  S=T=131,072 tokens, pools of 4 (32,768 pools), H=32,
                    D=128, K=2,048 positions = 512 pools, 2,051 output slots;
                    pool coefficients c ~ U(0, 0.5).
  long_1m_fp8       T=1,048,576 keys, the last 16,384 positions as queries,
                    H=64, D=128, K=2,048, FP8 e4m3 q and k with per-row FP32
                    scales (amax / 448).
  pooled_tail_64k   the pooled workload at S=T=65,536 (a profiling-sized case).
  long_1m_fp8_s2k   the FP8 workload with only the last 2,048 positions as
                    queries (a profiling-sized case).
  decode_1m_s16     16 query rows at the end of T=1,048,576 keys (a decode step
                    of 16 sequences' worth of indexer queries against one long
                    context), H=64, D=128, K=2,048, bf16: the split key-range
                    path.  Not one of the configurations the pages quote.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

TOKEN, COMPRESSED, POOLED = 0, 1, 2


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    S: int
    T: int
    H: int
    D: int
    K: int
    visibility: int = TOKEN
    ratio: int = 1
    dtype: str = "bf16"          # storage of q and k: "bf16" or "fp8"
    q_pos0: int = 0
    seed: int = 0
    values: str = "gauss"        # "gauss", "int", or "corr" (correlated heads, w >= 0)
    pair_overlap: bool = False   # the step also counts shared indices of adjacent query pairs

    def problem(self) -> dict:
        return dict(S=self.S, T=self.T, H=self.H, D=self.D, K=self.K,
                    visibility=self.visibility, ratio=self.ratio,
                    dtype=self.dtype, q_pos0=self.q_pos0)

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny_int_512": Workload("tiny_int_512", S=512, T=512, H=4, D=64, K=64,
                             seed=0, values="int"),
    "dsa_prefill_64k": Workload("dsa_prefill_64k", S=65536, T=65536, H=64,
                                D=128, K=2048, seed=1),
    "dsa_prefill_16k": Workload("dsa_prefill_16k", S=16384, T=16384, H=64,
                                D=128, K=2048, seed=5),
    "csa_m4_256k": Workload("csa_m4_256k", S=262144, T=65536, H=64, D=128,
                            K=2048, visibility=COMPRESSED, ratio=4, seed=2),
    "pooled_tail_128k": Workload("pooled_tail_128k", S=131072, T=131072, H=32,
                                 D=128, K=2048, visibility=POOLED, ratio=4,
                                 seed=3),
    "long_1m_fp8": Workload("long_1m_fp8", S=16384, T=1048576, H=64, D=128,
                            K=2048, dtype="fp8", q_pos0=1048576 - 16384,
                            seed=4, pair_overlap=True),
    "pooled_tail_64k": Workload("pooled_tail_64k", S=65536, T=65536, H=32,
                                D=128, K=2048, visibility=POOLED, ratio=4,
                                seed=7),
    "long_1m_fp8_s2k": Workload("long_1m_fp8_s2k", S=2048, T=1048576, H=64,
                                D=128, K=2048, dtype="fp8",
                                q_pos0=1048576 - 2048, seed=8),
    "decode_1m_s16": Workload("decode_1m_s16", S=16, T=1048576, H=64, D=128,
                              K=2048, q_pos0=1048576 - 16, seed=6),
}


def _quantise_e4m3_rows(x: torch.Tensor):
    """Per-row FP8 e4m3 quantisation of the last dimension: scale = amax/448
    (1 where a row is all zero), codes = e4m3(clamp(x / scale, +-448))."""
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    y = (x / scale.unsqueeze(-1)).clamp_(-448.0, 448.0)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale.to(torch.float32)


def _randn(shape, gen, device, chunk_rows=1 << 14):
    """Standard normal fp32 in row chunks (bounded temporary memory)."""
    out = torch.empty(shape, dtype=torch.float32, device=device)
    flat = out.view(shape[0], -1)
    for r0 in range(0, shape[0], chunk_rows):
        r1 = min(shape[0], r0 + chunk_rows)
        flat[r0:r1].normal_(generator=gen)
    return out


def generate(wl: Workload, device="cpu") -> dict:
    """Draw the workload's inputs on `device` with a generator seeded by wl.seed.

    Returns a dict of tensors:
      q [S, H, D] bf16 or uint8 (e4m3 codes), k [T, D] likewise,
      w [S, H] float32, q_scale [S, H] / k_scale [T] float32 for fp8 (else
      None), pool_coef [ratio, D] bf16 for POOLED (else None).
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed)
    out = dict(q_scale=None, k_scale=None, pool_coef=None)
    if wl.values == "int":
        out["q"] = torch.randint(-3, 4, (wl.S, wl.H, wl.D), generator=gen,
                                 device=device).to(torch.bfloat16)
        out["k"] = torch.randint(-3, 4, (wl.T, wl.D), generator=gen,
                                 device=device).to(torch.bfloat16)
        out["w"] = torch.randint(-2, 3, (wl.S, wl.H), generator=gen,
                                 device=device).to(torch.float32)
    else:
        q = _randn((wl.S, wl.H, wl.D), gen, device)
        k = _randn((wl.T, wl.D), gen, device)
        if wl.values == "corr":
            # structured heads: every head of a query is one shared direction
            # plus 1% noise (what lets a score certificate prune keys)
            z = _randn((wl.S, 1, wl.D), gen, device)
            q.mul_(0.01).add_(z)
        if wl.dtype == "fp8":
            out["q"], out["q_scale"] = _quantise_e4m3_rows(q)
            out["k"], out["k_scale"] = _quantise_e4m3_rows(k)
        else:
            out["q"] = q.to(torch.bfloat16)
            out["k"] = k.to(torch.bfloat16)
        del q, k
        w = _randn((wl.S, wl.H), gen, device) * (1.0 / math.sqrt(wl.H))
        out["w"] = (w.abs() if wl.values == "corr" else w).to(torch.float32)
    if wl.visibility == POOLED:
        if wl.values == "int":   # integer pooled keys: every score exact in FP32
            c = torch.randint(0, 2, (wl.ratio, wl.D), generator=gen, device=device,
                              dtype=torch.int32).to(torch.float32)
        else:
            c = torch.rand((wl.ratio, wl.D), generator=gen, device=device,
                           dtype=torch.float32) * 0.5
        out["pool_coef"] = c.to(torch.bfloat16)
    return out


def index_rows(S: int, width: int, universe: int, seed: int):
    """Seeded rows shaped like the indexer's output, for the pair steps:
    row r holds len[r] distinct ascending KV indices below `universe`, then -1
    padding.  Lengths cover 0 and width; pair 1 has two identical rows, pair 2
    two disjoint rows, and the other odd rows re-use about three quarters of
    their partner's indices (the high-overlap regime the pair steps target).
    Returns numpy int32 arrays idx [S, width] and len [S]."""
    import numpy as np
    rng = np.random.default_rng(seed)
    idx = np.full((S, width), -1, dtype=np.int32)
    ln = np.zeros(S, dtype=np.int32)
    for r in range(S):
        n = int(rng.integers(0, width + 1)) if r > 5 else [0, width, width, width, width // 2, width // 2][r]
        if r in (3,):
            row = idx[2, : ln[2]]
        elif r == 5:
            taken = set(idx[4, : ln[4]].tolist())
            free = np.array([v for v in range(universe) if v not in taken])
            row = np.sort(rng.choice(free, size=min(n, free.size), replace=False))
        elif r % 2 == 1 and ln[r - 1] > 0:
            prev = idx[r - 1, : ln[r - 1]]
            keep = prev[rng.random(prev.size) < 0.75]
            extra = rng.choice(universe, size=max(n - keep.size, 0), replace=False)
            row = np.unique(np.concatenate([keep, extra]))[:width]
        else:
            row = np.sort(rng.choice(universe, size=n, replace=False))
        idx[r, : row.size] = row
        ln[r] = row.size
    return idx, ln


def sample_rows(wl: Workload, n: int = 1024, seed: int = 12345) -> np.ndarray:
    """Seeded query rows for the oracle: the first 4 rows, rows whose global
    position is near K (K-2 .. K+1) and near the first pool boundaries, the
    last row, and the rest drawn uniformly without replacement; ascending."""
    S = wl.S
    special = {0, 1, 2, 3, S - 1, S - 2}
    for g in range(wl.K - 2, wl.K + 2):
        special.add(g - wl.q_pos0)
    m = max(wl.ratio, 1)
    for g in (m - 2, m - 1, m, 2 * m - 1, 2 * m, 4 * wl.K - 1, 4 * wl.K):
        special.add(g - wl.q_pos0)
    special = {t for t in special if 0 <= t < S}
    rng = np.random.default_rng(seed)
    rest = n - len(special)
    pool = np.setdiff1d(np.arange(S), np.fromiter(special, dtype=np.int64))
    if rest > 0 and pool.size:
        extra = rng.choice(pool, size=min(rest, pool.size), replace=False)
    else:
        extra = np.zeros(0, dtype=np.int64)
    rows = np.union1d(np.fromiter(special, dtype=np.int64), extra)
    return rows.astype(np.int64)


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    """Storage bits of a tensor as numpy (bf16 -> uint16, uint8 unchanged,
    float32 unchanged)."""
    if t is None:
        return None
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()
