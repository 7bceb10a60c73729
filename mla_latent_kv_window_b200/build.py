"""Build step of libmla.so: one nvcc invocation, sm_100a only, output next to this file.

build(debug=True) makes libmla_debug.so from the same sources with MLA_DEBUG defined: bounds
checks on every computed global index (a violation records MLA_ERR_BOUNDS in the status word and
skips the access) and guard bands after every device buffer, checked by mla_cache_sync.  It
stands in for a memory checker; select it with MLA_LIBRARY=<path> before loading the binding."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libmla.so")
LIB_DEBUG = os.path.join(HERE, "libmla_debug.so")
SOURCES = [os.path.join(HERE, "csrc", "mla_api.cu")]
DEPS = SOURCES + [os.path.join(HERE, "csrc", f) for f in ("ptx.cuh", "gemm_tc.cuh", "query_proj.cuh", "window_attn.cuh", "dense_attn.cuh")] + \
    [os.path.join(ROOT, "include", "mla.h")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    raise RuntimeError("nvcc not found")


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(lib):
        return lib
    tmp = f"{lib}.{os.getpid()}.tmp"
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-cudart", "static", "-I", os.path.join(ROOT, "include"),
           "-o", tmp] + (["-DMLA_DEBUG"] if debug else []) + SOURCES
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
