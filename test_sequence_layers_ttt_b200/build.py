"""Build libttt_b200.so (the C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libttt_b200.so")
# the same library with the clock64 timeline stamps compiled in (timeline.py reads them)
TIMELINE_LIB = os.path.join(PKG, "libttt_b200_timeline.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + [
        os.path.join(ROOT, "include", "ttt.h")]


def build(force: bool = False, verbose: bool = False, timeline: bool = False) -> str:
    out = TIMELINE_LIB if timeline else LIB
    stale = (not os.path.exists(out)) or any(os.path.getmtime(p) > os.path.getmtime(out) for p in deps())
    if not (force or stale):
        return out
    nvcc = os.environ.get("NVCC", "nvcc")
    if not os.path.isabs(nvcc) and os.path.exists("/usr/local/cuda/bin/nvcc"):
        nvcc = "/usr/local/cuda/bin/nvcc"
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, *(["-DTTT_TIMELINE"] if timeline else []), "-I", os.path.join(ROOT, "include"),
           "-o", tmp, *sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, timeline="--timeline" in sys.argv))
