"""Builds libsage.so in-tree with nvcc for sm_100a (no JIT cache, no pip install)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SOURCES = ["api.cu", "prepass.cu", "attention.cu", "noalloc.cu", "calib.cu", "linear.cu", "ulysses.cu", "diag.cu"]
HEADERS = ["internal.h", "sm100.cuh"]
LIB_PATH = os.path.join(HERE, "libsage.so")
# the same sources with device-side bounds checks (SAGE_DEBUG, see include/sage.h)
DEBUG_LIB_PATH = os.path.join(HERE, "libsage_debug.so")
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale(path: str) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "sage.h"),
                                                                  os.path.abspath(__file__)]
    return any(os.path.getmtime(p) > t for p in deps)


def _compile(path: str, extra: list, verbose: bool):
    tmp = path + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, *extra, "-o", tmp] + [os.path.join(CSRC, f) for f in SOURCES]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd, cwd=HERE)
    os.replace(tmp, path)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compiles csrc/*.cu into libsage.so next to this file if it is missing or stale
    (debug=True: libsage_debug.so, the same sources with -DSAGE_DEBUG)."""
    path, extra = (DEBUG_LIB_PATH, ["-DSAGE_DEBUG"]) if debug else (LIB_PATH, [])
    if force or _stale(path):
        _compile(path, extra, verbose)
    return path


def build_all(force: bool = False, verbose: bool = False) -> list:
    """Both libraries; the two compilations run side by side."""
    import concurrent.futures as cf
    with cf.ThreadPoolExecutor(2) as ex:
        futs = [ex.submit(build, force, verbose, dbg) for dbg in (False, True)]
        return [f.result() for f in futs]


if __name__ == "__main__":
    print(build_all(force="--force" in sys.argv, verbose=True))
