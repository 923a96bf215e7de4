"""Build ``libthrift.so`` (the C-ABI CUDA library) in-tree with nvcc for sm_100a,
and ``probe/libthrift_probe.so``, the benchmark's tensor-pipe rate probe (a
measurement helper kept out of the library's ABI)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libthrift.so")
PROBE_DIR = os.path.join(HERE, "probe")
PROBE_LIB = os.path.join(PROBE_DIR, "libthrift_probe.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr"]


def sources(src_dir=CSRC):
    return sorted(glob.glob(os.path.join(src_dir, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(HERE, "..", "include", "*.h")))


def up_to_date(lib=LIB, src_dir=CSRC) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in sources(src_dir) + headers())


def _link(lib, src_dir, tag, verbose):
    objs = []
    build_dir = os.path.join(HERE, "_build", tag)
    os.makedirs(build_dir, exist_ok=True)
    for src in sources(src_dir):
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        cmd = [NVCC, *FLAGS, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.check_call(cmd)
        objs.append(obj)
    subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", *objs, "-o", lib])


def build(force: bool = False, verbose: bool = False) -> str:
    """Build both libraries when a source or header is newer; returns LIB."""
    if force or not up_to_date():
        _link(LIB, CSRC, "lib", verbose)
    if force or not up_to_date(PROBE_LIB, PROBE_DIR):
        _link(PROBE_LIB, PROBE_DIR, "probe", verbose)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
