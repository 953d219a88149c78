"""Build libpisa.so (the CUDA library behind the C ABI in include/pisa.h).

    python -m block_sparse_attention_stats_b200.build [--verbose-ptxas]

Compiles the single translation unit csrc/pisa_api.cu for sm_100a with nvcc
and writes libpisa.so next to this file (in-tree, so it travels with the
repository snapshot).  Rebuilds only when a source or header is newer than the
library, unless force=True.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libpisa.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    if os.path.exists(cand):
        return cand
    p = shutil.which("nvcc")
    if not p:
        raise RuntimeError("nvcc not found (set CUDA_HOME)")
    return p


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, ptxas_verbose: bool = False, log: str = "") -> str:
    if not force and not needs_build():
        return LIB
    cmd = [_nvcc(), *ARCH_FLAGS, "-O3", "-std=c++17", "-lineinfo", "--shared",
           "-Xcompiler", "-fPIC", "-cudart", "static", "-I", INCLUDE, "-I", CSRC,
           "-o", LIB + ".tmp", os.path.join(CSRC, "pisa_api.cu")]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    if ptxas_verbose:
        if log:
            with open(log, "w") as f:
                f.write(r.stderr)
        else:
            sys.stderr.write(r.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
