"""Build libeva_vq.so (the C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libeva_vq.so")
CHECKED_LIB = os.path.join(HERE, "libeva_vq_checked.so")   # device-side bounds checks
TIMELINE_LIB = os.path.join(HERE, "libeva_vq_timeline.so") # per-CTA phase timestamps
NAIVE_LIB = os.path.join(HERE, "libeva_vq_naive.so")       # naive [w][c] image layout (bank-conflict ablation)
SOURCES = [os.path.join(HERE, "csrc", "eva_vq.cu")]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libeva_vq.so")


def _inputs():
    return SOURCES + glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + glob.glob(os.path.join(HERE, "csrc", "*.h")) + \
        [os.path.join(ROOT, "include", "eva_vq.h")]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, checked: bool = False,
          timeline: bool = False, naive: bool = False) -> str:
    """Compile the library; checked=True builds the variant with device-side
    bounds checks (EVA_DEVICE_CHECKS), timeline=True the one that stamps each
    CTA's phases (EVA_TIMELINE), naive=True the one whose one-token image uses
    the naive row-per-sub-vector layout (EVA_NAIVE_OC_LAYOUT, to measure the
    bank conflicts the shipped layout avoids).  All three are diagnostics
    builds."""
    lib = CHECKED_LIB if checked else (TIMELINE_LIB if timeline else (NAIVE_LIB if naive else LIB))
    if not force and up_to_date(lib):
        return lib
    extra = ["-DEVA_DEVICE_CHECKS"] if checked else (["-DEVA_TIMELINE"] if timeline else
                                                      (["-DEVA_NAIVE_OC_LAYOUT"] if naive else []))
    cmd = [_nvcc(), *NVCC_FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-o", lib + ".tmp", *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, checked="--checked" in sys.argv,
                timeline="--timeline" in sys.argv, naive="--naive" in sys.argv))
