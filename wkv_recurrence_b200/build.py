"""Build libwkv.so in-tree with nvcc for sm_100a (Blackwell B200).

    python -m wkv_recurrence_b200.build            # build if sources changed
    python -m wkv_recurrence_b200.build --force    # always rebuild
    python -m wkv_recurrence_b200.build --debug    # also the bounds-checked libwkv_debug.so

nvcc cross-compiles, so this runs on a machine without a GPU. The
bounds-checked variant (-DWKV_DEBUG) checks the indices of the kernels'
stores and workspace accesses and reports a violation through the status
word (WKV_ERR_BOUNDS from wkv_query_status) instead of touching memory; the
binding loads it instead of libwkv.so when WKV_LIBRARY=debug is set.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC_DIR = os.path.join(HERE, "csrc")
MAIN = os.path.join(SRC_DIR, "wkv_api.cu")
HOST = os.path.join(SRC_DIR, "wkv_host.cpp")  # host-side streaming of host-resident sequences
LIB = os.path.join(HERE, "_build", "libwkv.so")
LIB_DEBUG = os.path.join(HERE, "_build", "libwkv_debug.so")
HEADER = os.path.join(ROOT, "include", "wkv.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-Xcompiler", "-Wall",
]


def _sources():
    return sorted(glob.glob(os.path.join(SRC_DIR, "*.cu")) + glob.glob(os.path.join(SRC_DIR, "*.cuh"))
                  + glob.glob(os.path.join(SRC_DIR, "*.cpp")) + [HEADER])


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def build(force: bool = False, verbose: bool = False, extra_flags=(), debug: bool = False) -> str:
    out = LIB_DEBUG if debug else LIB
    newest = max(os.path.getmtime(p) for p in _sources())
    if not force and os.path.exists(out) and os.path.getmtime(out) >= newest:
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *(["-DWKV_DEBUG"] if debug else []), *extra_flags, "-o", tmp, MAIN, HOST]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build_all(force: bool = False, verbose: bool = False):
    """Both variants, compiled concurrently."""
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(2) as ex:
        futs = [ex.submit(build, force, verbose, (), d) for d in (False, True)]
        return [f.result() for f in futs]


if __name__ == "__main__":
    if "--debug" in sys.argv:
        print(build_all(force="--force" in sys.argv, verbose=True))
    else:
        print(build(force="--force" in sys.argv, verbose=True))
