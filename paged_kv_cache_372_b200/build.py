"""Builds libpa_b200.so, the sm_100a CUDA library behind include/pa.h, in-tree.

    python -m paged_kv_cache_372_b200.build [--force] [--verbose]

nvcc compiles csrc/pa_api.cu (which includes the kernel headers) and
csrc/pa_noalloc.cu for sm_100a only. The result lands in ``_lib/`` next to this
file, so it travels with the source tree.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(HERE, "_lib")
LIB = os.path.join(LIB_DIR, "libpa_b200.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libpa_b200")
    return path


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(INCLUDE, "pa.h")])


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          out: str | None = None) -> str:
    """Compile when a source is newer than the library (or force). `extra` adds nvcc
    flags (e.g. -DPA_DECODE_STAGES=6); `out` writes the library elsewhere."""
    target = out or LIB
    if not force and out is None and not stale():
        return LIB
    os.makedirs(os.path.dirname(target), exist_ok=True)
    tmp = target + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE,
           os.path.join(CSRC, "pa_api.cu"), os.path.join(CSRC, "pa_noalloc.cu"), "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    cmd += extra or []
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        print(res.stdout + res.stderr)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
