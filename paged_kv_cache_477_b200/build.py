"""Build libpagedkv.so in-tree with nvcc for sm_100a.

    python -m paged_kv_cache_477_b200.build [--force] [-v]

The library is one translation unit (csrc/pagedkv_api.cu includes the kernel
headers) so that all kernels share the device error word.  cudart is linked
statically; the library allocates no device memory of its own.
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
SRC = os.path.join(CSRC, "pagedkv_api.cu")
LIB = os.path.join(HERE, "libpagedkv.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps():
    return ([SRC] + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.hpp")) +
            [os.path.join(ROOT, "include", "pagedkv.h")])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in _deps())


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          out: str | None = None) -> str:
    """Compile the library (to ``out``, default the in-tree libpagedkv.so)."""
    target = out or LIB
    if not force and out is None and up_to_date():
        return LIB
    cmd = [nvcc_path(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
           "-shared", "-Xcompiler", "-fPIC,-O2", "-I", os.path.join(ROOT, "include"),
           "-o", target + ".tmp", SRC]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    if extra:
        cmd += list(extra)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        print(res.stdout + res.stderr)
    os.replace(target + ".tmp", target)
    return target


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
