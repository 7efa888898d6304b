"""Build libspecverify.so (and its bounds-checked twin libspecverify_debug.so)
in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = [os.path.join(PKG, "csrc", "spec_verify.cu")]
HDR = os.path.join(ROOT, "include", "spec_verify.h")
OUT = os.path.join(PKG, "libspecverify.so")
OUT_DEBUG = os.path.join(PKG, "libspecverify_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
]
DEBUG_FLAGS = ["-DSPEC_DEBUG_BOUNDS"]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale(out: str = OUT) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(p) > t for p in SRC + [HDR, __file__])


def _cmd(out: str, extra) -> list:
    return [nvcc(), *NVCC_FLAGS, *extra, "-I", os.path.join(ROOT, "include"), *SRC, "-o", out + ".tmp"]


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Compile the library (and, with ``debug``, the bounds-checked one) when a
    source is newer than it; the two compile in parallel.  Returns the path of
    the library."""
    jobs = [(o, x) for o, x in [(OUT, []), (OUT_DEBUG, DEBUG_FLAGS)] if (o == OUT or debug) and (force or stale(o))]
    procs = []
    for out, extra in jobs:
        cmd = _cmd(out, extra)
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        procs.append((out, subprocess.Popen(cmd)))
    failed = [out for out, p in procs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, f"nvcc ({', '.join(failed)})")
    for out, _ in procs:
        os.replace(out + ".tmp", out)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
