"""Thin ctypes binding over libhwr_indexer.so (include/hwr_indexer.h).

The functions named like the C entry points marshal arguments only: torch
tensors become raw device pointers, torch streams become cudaStream_t.  Every
step of the indexer runs in the library's kernels; there is no fallback.  If the
library is missing, importing this module raises.

`topk(...)` is the convenience call most users want: it allocates outputs and
workspace with torch (plumbing) and calls indexer_topk.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# HWR_INDEXER_LIB may point at another build of the same library (same ABI)
LIB_PATH = os.environ.get("HWR_INDEXER_LIB") or os.path.join(_HERE, "libhwr_indexer.so")

TOKEN, COMPRESSED, POOLED = 0, 1, 2
BF16, FP8_E4M3 = 0, 1
FLAG_PRUNE = 1
FLAG_TEST_WAIT_TIMEOUT = 1 << 30   # test hook: the kernel's wait-timeout path (outputs not valid)

STATUS_NAMES = {0: "INDEXER_OK", 1: "INDEXER_EINVAL", 2: "INDEXER_EWORKSPACE",
                3: "INDEXER_EUNSUPPORTED", 4: "INDEXER_ECUDA", 5: "INDEXER_EDEVICE"}

# every symbol include/hwr_indexer.h declares
EXPORTS = ("indexer_out_width", "indexer_workspace_bytes", "indexer_partition_rows",
           "indexer_topk", "indexer_topk_noalloc", "indexer_noalloc_read_status",
           "indexer_host_workspace_bytes", "indexer_topk_host",
           "indexer_docs_workspace_bytes", "indexer_topk_docs",
           "indexer_padded_workspace_bytes", "indexer_topk_padded",
           "indexer_witness_workspace_bytes", "indexer_topk_witness",
           "indexer_pool_keys",
           "indexer_pair_overlap", "indexer_pair_regions", "indexer_read_status", "indexer_read_prune_counters",
           "indexer_status_string",
           "indexer_abi_version", "indexer_build_info")


class IndexerError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        msg = _lib.indexer_status_string(status).decode()
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)} ({msg})")


class Problem(ctypes.Structure):
    """Mirror of indexer_problem."""
    _fields_ = [("S", ctypes.c_int64), ("T", ctypes.c_int64), ("H", ctypes.c_int32),
                ("D", ctypes.c_int32), ("q_pos0", ctypes.c_int64), ("visibility", ctypes.c_int32),
                ("ratio", ctypes.c_int32), ("K", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("flags", ctypes.c_int32), ("reserved", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m head_weighted_relu_b200.build` "
            "(the indexer has no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    lib.indexer_build_info.argtypes = []
    lib.indexer_build_info.restype = ctypes.c_char_p
    if "HWR_INDEXER_LIB" not in os.environ:
        # the library must come from the sources beside it (a stale build would
        # otherwise pass unnoticed)
        from . import build as _build
        want = "source_sha256=" + _build.source_hash()
        got = lib.indexer_build_info().decode()
        if got != want:
            raise ImportError(f"{LIB_PATH} was built from other sources ({got[:30]}...); "
                              "rebuild it with `python -m head_weighted_relu_b200.build`")
    P = ctypes.POINTER(Problem)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    lib.indexer_out_width.argtypes = [P, ctypes.POINTER(i32)]
    lib.indexer_workspace_bytes.argtypes = [P, ctypes.POINTER(ctypes.c_size_t)]
    lib.indexer_partition_rows.argtypes = [P, i32, ctypes.POINTER(i64)]
    lib.indexer_topk.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.indexer_topk_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.indexer_noalloc_read_status.argtypes = [ctypes.POINTER(i32), vp]
    lib.indexer_host_workspace_bytes.argtypes = [P, ctypes.POINTER(ctypes.c_size_t)]
    lib.indexer_topk_host.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.indexer_docs_workspace_bytes.argtypes = [P, vp, i32, ctypes.POINTER(ctypes.c_size_t)]
    lib.indexer_topk_docs.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.indexer_padded_workspace_bytes.argtypes = [P, vp, i32, i64, ctypes.POINTER(ctypes.c_size_t)]
    lib.indexer_topk_padded.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, i32, i64, vp, vp, vp, vp,
                                        ctypes.c_size_t, vp]
    lib.indexer_witness_workspace_bytes.argtypes = [P, i64, ctypes.POINTER(ctypes.c_size_t)]
    lib.indexer_topk_witness.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, i64, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.indexer_pool_keys.argtypes = [vp, i64, i32, vp, i32, vp, vp]
    lib.indexer_pair_overlap.argtypes = [vp, vp, i64, i32, vp, vp]
    lib.indexer_pair_regions.argtypes = [vp, vp, i64, i32, vp, vp, vp, vp, vp]
    lib.indexer_read_status.argtypes = [vp, ctypes.POINTER(i32), vp]
    lib.indexer_read_prune_counters.argtypes = [vp, ctypes.POINTER(ctypes.c_uint64), vp]
    lib.indexer_status_string.argtypes = [ctypes.c_int]
    lib.indexer_status_string.restype = ctypes.c_char_p
    lib.indexer_abi_version.argtypes = []
    for name in EXPORTS:
        if name not in ("indexer_status_string", "indexer_build_info"):
            getattr(lib, name).restype = ctypes.c_int
    return lib


_lib = _load()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, status):
    if status != 0:
        raise IndexerError(fn, status)


def make_problem(S, T, H, D, K, visibility=TOKEN, ratio=1, dtype=BF16, q_pos0=0,
                 prune=False, flags=0) -> Problem:
    if isinstance(dtype, str):
        dtype = {"bf16": BF16, "fp8": FP8_E4M3}[dtype]
    return Problem(S=S, T=T, H=H, D=D, q_pos0=q_pos0, visibility=visibility, ratio=ratio,
                   K=K, dtype=dtype, flags=(FLAG_PRUNE if prune else 0) | flags, reserved=0)


def indexer_out_width(problem: Problem) -> int:
    w = ctypes.c_int32()
    _check("indexer_out_width", _lib.indexer_out_width(ctypes.byref(problem), ctypes.byref(w)))
    return w.value


def indexer_workspace_bytes(problem: Problem) -> int:
    n = ctypes.c_size_t()
    _check("indexer_workspace_bytes",
           _lib.indexer_workspace_bytes(ctypes.byref(problem), ctypes.byref(n)))
    return n.value


def indexer_partition_rows(problem: Problem, n_parts: int) -> list:
    """Row bounds [0, ..., S] splitting the problem's query rows into n_parts
    parts of about equal visible-pair count (one part per GPU)."""
    b = (ctypes.c_int64 * (n_parts + 1))()
    _check("indexer_partition_rows", _lib.indexer_partition_rows(ctypes.byref(problem), n_parts, b))
    return [int(x) for x in b]


def indexer_topk(problem, q, k, w, q_scale, k_scale, pool_coef, out_idx, out_len, out_score,
                 workspace, stream=None):
    _check("indexer_topk", _lib.indexer_topk(
        ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(w), _ptr(q_scale), _ptr(k_scale),
        _ptr(pool_coef), _ptr(out_idx), _ptr(out_len), _ptr(out_score), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)))


def indexer_witness_workspace_bytes(problem: Problem, n_seeds: int) -> int:
    n = ctypes.c_size_t()
    _check("indexer_witness_workspace_bytes",
           _lib.indexer_witness_workspace_bytes(ctypes.byref(problem), ctypes.c_int64(n_seeds), ctypes.byref(n)))
    return n.value


def indexer_topk_witness(problem, q, k, w, q_scale, k_scale, pool_coef, seeds, out_idx, out_len, out_score,
                         workspace, stream=None):
    """indexer_topk starting from a seed threshold: seeds is a [S, n] int32
    device tensor of key indices per query (e.g. the previous decode step's
    out_idx), -1 or invisible entries ignored.  Same result as indexer_topk."""
    if seeds.dtype != torch.int32 or seeds.dim() != 2 or not seeds.is_contiguous():
        raise ValueError("seeds must be a contiguous [S, n] int32 tensor")
    _check("indexer_topk_witness", _lib.indexer_topk_witness(
        ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(w), _ptr(q_scale), _ptr(k_scale),
        _ptr(pool_coef), _ptr(seeds), ctypes.c_int64(seeds.shape[1]), _ptr(out_idx), _ptr(out_len),
        _ptr(out_score), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)))


def indexer_host_workspace_bytes(problem: Problem) -> int:
    n = ctypes.c_size_t()
    _check("indexer_host_workspace_bytes",
           _lib.indexer_host_workspace_bytes(ctypes.byref(problem), ctypes.byref(n)))
    return n.value


def indexer_topk_host(problem, q, k, w, q_scale, k_scale, pool_coef, out_idx, out_len, out_score,
                      workspace, stream=None):
    """indexer_topk on host tensors (pinned for the copies to overlap): inputs and
    outputs live in host memory, `workspace` is a device buffer of
    indexer_host_workspace_bytes bytes.  Ordered on `stream`; synchronise it
    before reading the outputs."""
    _check("indexer_topk_host", _lib.indexer_topk_host(
        ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(w), _ptr(q_scale), _ptr(k_scale),
        _ptr(pool_coef), _ptr(out_idx), _ptr(out_len), _ptr(out_score), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def _bounds(doc_bounds):
    import numpy as np
    b = np.ascontiguousarray(np.asarray(doc_bounds, dtype=np.int64))
    return b, ctypes.c_void_p(b.ctypes.data), len(b) - 1


def indexer_docs_workspace_bytes(problem: Problem, doc_bounds) -> int:
    b, ptr, n = _bounds(doc_bounds)
    out = ctypes.c_size_t()
    _check("indexer_docs_workspace_bytes",
           _lib.indexer_docs_workspace_bytes(ctypes.byref(problem), ptr, n, ctypes.byref(out)))
    return out.value


def indexer_topk_docs(problem, q, k, w, q_scale, k_scale, pool_coef, doc_bounds, out_idx, out_len,
                      out_score, workspace, stream=None):
    """indexer_topk for a packed batch of documents: doc_bounds (host, n_docs + 1
    token positions) splits the tokens; a query sees only its own document."""
    b, ptr, n = _bounds(doc_bounds)
    _check("indexer_topk_docs", _lib.indexer_topk_docs(
        ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(w), _ptr(q_scale), _ptr(k_scale), _ptr(pool_coef),
        ptr, n, _ptr(out_idx), _ptr(out_len), _ptr(out_score), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def indexer_padded_workspace_bytes(problem: Problem, seq_lens, stride: int) -> int:
    b, ptr, n = _bounds(seq_lens)
    out = ctypes.c_size_t()
    _check("indexer_padded_workspace_bytes",
           _lib.indexer_padded_workspace_bytes(ctypes.byref(problem), ptr, n + 1, stride, ctypes.byref(out)))
    return out.value


def indexer_topk_padded(problem, q, k, w, q_scale, k_scale, pool_coef, seq_lens, stride, out_idx, out_len,
                        out_score, workspace, stream=None):
    """indexer_topk for a padded batch: sequence b is rows b*stride ..
    b*stride + seq_lens[b] - 1 (seq_lens on the host); padding rows select
    nothing."""
    b, ptr, n = _bounds(seq_lens)
    _check("indexer_topk_padded", _lib.indexer_topk_padded(
        ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(w), _ptr(q_scale), _ptr(k_scale), _ptr(pool_coef),
        ptr, n + 1, stride, _ptr(out_idx), _ptr(out_len), _ptr(out_score), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def indexer_topk_noalloc(problem, q, k, w, q_scale, k_scale, pool_coef, out_idx, out_len,
                         out_score, stream=None):
    """indexer_topk without a workspace: for callers that cannot allocate device
    memory.  Scratch is the library's fixed 64 MiB device array; larger problems
    raise IndexerError (INDEXER_EWORKSPACE).  Calls share that array, so calls
    that could overlap on the GPU must be serialised."""
    _check("indexer_topk_noalloc", _lib.indexer_topk_noalloc(
        ctypes.byref(problem), _ptr(q), _ptr(k), _ptr(w), _ptr(q_scale), _ptr(k_scale),
        _ptr(pool_coef), _ptr(out_idx), _ptr(out_len), _ptr(out_score), _stream(stream)))


def indexer_noalloc_read_status(stream=None) -> int:
    """Status word of the last indexer_topk_noalloc call (read and cleared)."""
    f = ctypes.c_int32()
    _check("indexer_noalloc_read_status", _lib.indexer_noalloc_read_status(ctypes.byref(f), _stream(stream)))
    return f.value


def indexer_pool_keys(k, T_tokens, D, pool_coef, ratio, out_kp, stream=None):
    _check("indexer_pool_keys", _lib.indexer_pool_keys(
        _ptr(k), T_tokens, D, _ptr(pool_coef), ratio, _ptr(out_kp), _stream(stream)))


def indexer_pair_overlap(idx, lens, S, width, out_shared, stream=None):
    _check("indexer_pair_overlap", _lib.indexer_pair_overlap(
        _ptr(idx), _ptr(lens), S, width, _ptr(out_shared), _stream(stream)))


def indexer_pair_regions(idx, lens, S, width, out_shared, out_left, out_right, out_counts, stream=None):
    _check("indexer_pair_regions", _lib.indexer_pair_regions(
        _ptr(idx), _ptr(lens), S, width, _ptr(out_shared), _ptr(out_left), _ptr(out_right), _ptr(out_counts),
        _stream(stream)))


def indexer_read_status(workspace, stream=None) -> int:
    f = ctypes.c_int32()
    _check("indexer_read_status",
           _lib.indexer_read_status(_ptr(workspace), ctypes.byref(f), _stream(stream)))
    return f.value


def indexer_read_prune_counters(workspace, stream=None):
    """(pairs screened, pairs bounded below the threshold, pairs skipped) of the
    last call that used `workspace`."""
    c = (ctypes.c_uint64 * 3)()
    _check("indexer_read_prune_counters", _lib.indexer_read_prune_counters(
        _ptr(workspace), c, _stream(stream)))
    return tuple(int(x) for x in c)


def indexer_abi_version() -> int:
    return _lib.indexer_abi_version()


def indexer_build_info() -> str:
    """The build's identity: "source_sha256=<hash of the sources and flags>"."""
    return _lib.indexer_build_info().decode()


# ---------------------------------------------------------------------------
# Convenience layer (allocation through torch; compute through the library).
# ---------------------------------------------------------------------------

def _as_storage(x):
    """q / k storage as the library expects it: bf16, or e4m3 codes as uint8."""
    if x.dtype == torch.float8_e4m3fn:
        return x.view(torch.uint8)
    return x


def allocate(problem: Problem, device, with_scores=False):
    """Outputs and workspace for `problem` on `device` (torch allocations)."""
    width = indexer_out_width(problem)
    out_idx = torch.empty((problem.S, width), dtype=torch.int32, device=device)
    out_len = torch.empty((problem.S,), dtype=torch.int32, device=device)
    out_score = (torch.empty((problem.S, width), dtype=torch.float32, device=device)
                 if with_scores else None)
    ws = torch.empty((max(indexer_workspace_bytes(problem), 256),), dtype=torch.uint8, device=device)
    return out_idx, out_len, out_score, ws


def topk(q, k, w, K, visibility=TOKEN, ratio=1, q_pos0=0, q_scale=None, k_scale=None,
         pool_coef=None, with_scores=False, stream=None, buffers=None, prune=False):
    """Indexer top-K of every query row (prune=True: the lossless pruning stage).

    q [S, H, D] bf16 (or e4m3 / uint8 codes with q_scale [S, H]), k [T, D] likewise
    (k_scale [T]), w [S, H] float32.  Returns (idx [S, W] int32, len [S] int32) and,
    with_scores=True, also score [S, W] float32.
    """
    q, k = _as_storage(q), _as_storage(k)
    S, H, D = q.shape
    fp8 = q.dtype == torch.uint8
    prob = make_problem(S=S, T=k.shape[0], H=H, D=D, K=K, visibility=visibility,
                        ratio=ratio if visibility != TOKEN else 1,
                        dtype=FP8_E4M3 if fp8 else BF16, q_pos0=q_pos0, prune=prune)
    if buffers is None:
        buffers = allocate(prob, q.device, with_scores)
    out_idx, out_len, out_score, ws = buffers
    indexer_topk(prob, q.contiguous(), k.contiguous(), w.contiguous().float(),
                 None if q_scale is None else q_scale.contiguous().float(),
                 None if k_scale is None else k_scale.contiguous().float(),
                 None if pool_coef is None else pool_coef.contiguous(),
                 out_idx, out_len, out_score, ws, stream)
    if with_scores:
        return out_idx, out_len, out_score
    return out_idx, out_len


def pair_overlap(idx, lens, stream=None):
    """Exact |A_2p ∩ A_2p+1| for each non-overlapping adjacent pair of rows."""
    S, width = idx.shape
    out = torch.empty((S // 2,), dtype=torch.int32, device=idx.device)
    indexer_pair_overlap(idx.contiguous(), lens.contiguous(), S, width, out, stream)
    return out


def pair_regions(idx, lens, stream=None):
    """Shared, left-only and right-only KV indices of each adjacent query pair,
    each [S/2, width] (ascending, -1 padded), and their lengths [S/2, 3]."""
    S, width = idx.shape
    outs = [torch.empty((S // 2, width), dtype=torch.int32, device=idx.device) for _ in range(3)]
    counts = torch.empty((S // 2, 3), dtype=torch.int32, device=idx.device)
    indexer_pair_regions(idx.contiguous(), lens.contiguous(), S, width, *outs, counts, stream)
    return outs[0], outs[1], outs[2], counts


def pool_keys(k, pool_coef, ratio, stream=None):
    """Pooled keys kp [T // ratio, D] bf16 from token keys k [T, D]."""
    T, D = k.shape
    out = torch.empty((T // ratio, D), dtype=torch.bfloat16, device=k.device)
    indexer_pool_keys(k.contiguous(), T, D, pool_coef.contiguous(), ratio, out, stream)
    return out
