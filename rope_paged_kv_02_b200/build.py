"""Builds liblbm.so (the C ABI library) in-tree with nvcc for sm_100a.

    python -m rope_paged_kv_02_b200.build          # rebuild if any source is newer
    python -m rope_paged_kv_02_b200.build --force  # always rebuild

The library links the CUDA runtime statically and resolves the one driver entry point it
needs (cuTensorMapEncodeTiled) at run time, so it loads on a machine without a GPU driver.
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "liblbm.so")
SOURCES = ["pager.cpp", "rope.cu", "attn_tc.cu", "attn_simt.cu", "attn_static.cu", "lbm.cpp"]
HEADERS = ["pager.h", "lbm_internal.h"]

NVCC = os.environ.get("NVCC", "nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared",
]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps += [os.path.join(INCLUDE, "lbm.h"), os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every CUDA / C++ source into liblbm.so; returns its path."""
    if not force and not _stale():
        return LIB
    tmp = LIB + ".tmp"
    cmd = [NVCC, *FLAGS, "-I", INCLUDE, "-o", tmp] + [os.path.join(CSRC, f) for f in SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True, timeout=900)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
