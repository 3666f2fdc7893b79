"""Build libhwr_indexer.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m head_weighted_relu_b200.build [--verbose]

Each .cu under csrc/ is compiled to an object in parallel, then linked into
head_weighted_relu_b200/libhwr_indexer.so (static CUDA runtime, so the library
does not depend on the host program's runtime version).  A SHA-256 of the
sources and flags is compiled into the library (indexer_build_info) and
recorded beside it; a build whose recorded hash matches the sources is reused,
and the binding refuses to load a library built from other sources.
"""

from __future__ import annotations

import concurrent.futures as cf
import hashlib
import json
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libhwr_indexer.so")
INFO = os.path.join(PKG, "libhwr_indexer.build.json")   # the recorded build (not committed)
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def inputs() -> list:
    """Every file the library is compiled from."""
    paths = sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    paths.append(os.path.join(ROOT, "include", "hwr_indexer.h"))
    return sorted(paths)


def source_hash() -> str:
    """SHA-256 over the library's inputs (names and contents) and the compile
    flags: the identity of a build."""
    h = hashlib.sha256()
    for p in inputs():
        h.update(os.path.relpath(p, ROOT).encode() + b"\0")
        with open(p, "rb") as f:
            h.update(f.read())
        h.update(b"\0")
    h.update(" ".join(ARCH + FLAGS[:-2]).encode())
    return h.hexdigest()


def _recorded_hash():
    try:
        with open(INFO) as f:
            return json.load(f).get("source_sha256")
    except Exception:
        return None


def build(verbose: bool = False, force: bool = False) -> str:
    """Compile the library unless the recorded build already matches the
    current sources (by content hash, not by file times)."""
    digest = source_hash()
    if not force and os.path.exists(LIB) and _recorded_hash() == digest:
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    exe = nvcc()
    # the build's identity, compiled into the library (indexer_build_info)
    info_src = os.path.join(BUILD_DIR, "build_info.cu")
    with open(info_src, "w") as f:
        f.write('extern "C" const char* indexer_build_info(void) { return "source_sha256=%s"; }\n' % digest)

    def compile_one(src):
        obj = os.path.join(BUILD_DIR, os.path.basename(src) + ".o")
        cmd = [exe, *ARCH, *FLAGS, "-c", src, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stdout + r.stderr

    with cf.ThreadPoolExecutor(max_workers=len(sources()) + 1) as ex:
        results = list(ex.map(compile_one, sources() + [info_src]))
    if verbose:
        for _, log in results:
            if log.strip():
                print(log)
    objs = [o for o, _ in results]
    tmp = LIB + ".tmp"
    cmd = [exe, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    with open(INFO, "w") as f:
        json.dump({"source_sha256": digest, "nvcc": exe, "flags": ARCH + FLAGS[:-2]}, f)
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force="--force" in sys.argv))
