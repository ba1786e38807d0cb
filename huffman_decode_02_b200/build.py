"""Builds libdf11.so in-tree with nvcc for sm_100a.

Sources: every csrc/*.cu and csrc/*.cpp (host encoder / planner, decode and
row-gather kernels, device encoder, consumer GEMM).  The CUDA runtime is
linked statically, so the library needs only the driver.

`build(debug=True)` builds libdf11_debug.so from the same sources with
DF11_DEBUG_CHECKS: every data-dependent shared-memory index and global
store address of the decode kernels is checked before the access (a failed
check skips it and is counted; read with df11_debug_bounds_errors).  It is
for tests; the product library is libdf11.so.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(HERE, "libdf11.so")
DEBUG_LIB_PATH = os.path.join(HERE, "libdf11_debug.so")

NVCC_FLAGS = [
    "-std=c++17", "-O3", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-O3", "-Xcompiler", "-pthread",
    "-shared", "-cudart", "static",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _stale(path: str) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compiles every source to an object file (in parallel, one nvcc per
    source) under _build/, then links the shared library."""
    path = DEBUG_LIB_PATH if debug else LIB_PATH
    if not force and not _stale(path):
        return path
    tag = ("debug" if debug else "release") + f".{os.getpid()}"
    obj_dir = os.path.join(HERE, "_build")
    os.makedirs(obj_dir, exist_ok=True)
    extra = ["-DDF11_DEBUG_CHECKS"] if debug else []
    compile_flags = [f for f in NVCC_FLAGS if f != "-shared"]
    jobs = []
    for src in sources():
        obj = os.path.join(obj_dir, os.path.basename(src) + f".{tag}.o")
        jobs.append((obj, [_nvcc(), *compile_flags, *extra, "-I" + INCLUDE, "-I" + CSRC, "-c", src, "-o", obj]))
    procs = []
    for _, cmd in jobs:
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        procs.append(subprocess.Popen(cmd))
    failed = [cmd for (_, cmd), p in zip(jobs, procs) if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, failed[0])
    tmp = path + f".tmp{os.getpid()}"
    link = [_nvcc(), *NVCC_FLAGS, *[obj for obj, _ in jobs], "-o", tmp]
    if verbose:
        print(" ".join(link), file=sys.stderr)
    subprocess.check_call(link)
    for obj, _ in jobs:
        os.remove(obj)
    os.replace(tmp, path)
    return path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
