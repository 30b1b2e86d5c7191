"""Build libw4a16.so (the CUDA library behind include/w4a16.h) in-tree, and
its index-check twin libw4a16_debug.so (-DW4A16_DEBUG_BOUNDS: the decode
kernel checks every global and shared-memory access it makes against its
buffer and records a failure in the device status word instead of making
the access; same API).

nvcc cross-compiles for sm_100a without a GPU.  The libraries link the CUDA
runtime statically and export only the C entry points.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libw4a16.so")
LIB_DEBUG = os.path.join(HERE, "libw4a16_debug.so")
NVCC = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (sources() + glob.glob(os.path.join(CSRC, "*.cuh"))
            + [os.path.join(ROOT, "include", "w4a16.h")])


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def _command(lib: str, tmp: str, extra=None):
    cmd = [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC,-fvisibility=hidden", "-Xptxas", "-v",
           "-I", os.path.join(ROOT, "include"), "-o", tmp, *sources()]
    if lib == LIB_DEBUG:
        cmd[1:1] = ["-DW4A16_DEBUG_BOUNDS"]
    if extra:
        cmd[1:1] = list(extra)
    return cmd


def build(force: bool = False, verbose: bool = False, extra=None, debug: bool = True) -> str:
    """Build libw4a16.so and (debug=True) libw4a16_debug.so where stale, the
    two nvcc runs side by side.  Returns the path of libw4a16.so."""
    libs = [LIB] + ([LIB_DEBUG] if debug else [])
    todo = [lib for lib in libs if force or not up_to_date(lib)]
    runs = []
    for lib in todo:
        tmp = lib + f".tmp{os.getpid()}"
        cmd = _command(lib, tmp, extra)
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        runs.append((lib, tmp, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
    failed = []
    for lib, tmp, proc in runs:
        out, _ = proc.communicate()
        log = os.path.join(HERE, "_ptxas.log" if lib == LIB else "_ptxas_debug.log")
        with open(log, "w") as f:
            f.write(out)
        if proc.returncode != 0:
            sys.stderr.write(out)
            failed.append(os.path.basename(lib))
            if os.path.exists(tmp):
                os.remove(tmp)
        else:
            os.replace(tmp, lib)
    if failed:
        raise RuntimeError("nvcc failed building " + ", ".join(failed))
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
