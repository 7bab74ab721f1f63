"""Builds libpa.so (the CUDA kernels and their C ABI) in-tree for sm_100a.

    python -m paged_kv_cache_382_b200.build [--verbose]

nvcc compiles every ``csrc/*.cu`` for ``sm_100a`` only (and the host-only
``csrc/*.cpp``) and links one shared
library next to this file; the CUDA runtime is linked statically, so the
library needs nothing from the environment beyond the NVIDIA driver.
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_PATH = os.path.join(HERE, "libpa.so")
SOURCES = sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")) + glob.glob(os.path.join(HERE, "csrc", "*.cpp")))
DEPS = SOURCES + [os.path.abspath(__file__)] + sorted(glob.glob(os.path.join(HERE, "csrc", "*.cuh")) +
                        glob.glob(os.path.join(HERE, "csrc", "*.h")) +
                        glob.glob(os.path.join(HERE, "csrc", "*.map")) +
                        glob.glob(os.path.join(ROOT, "include", "*.h")))

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libpa.so")


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(p) <= t for p in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libpa.so if any source is newer than it; returns its path."""
    if not force and up_to_date():
        return LIB_PATH
    tmp = LIB_PATH + ".tmp"
    cmd = [nvcc_path(), "-O3", "-std=c++17", *ARCH_FLAGS, "-lineinfo",
           "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden", "-shared", "-I", os.path.join(ROOT, "include"),
           "-Xlinker", "--version-script=" + os.path.join(HERE, "csrc", "libpa.map"),
           "-o", tmp, *SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}) building libpa.so")
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB_PATH)
