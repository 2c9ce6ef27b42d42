"""Build libdstopk.so in-tree for sm_100a with nvcc (no JIT cache).

    python -m sparse_attention_top_ds_b200.build          # build if stale
    python -m sparse_attention_top_ds_b200.build --force  # always rebuild
"""

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
HEADER = os.path.join(ROOT, "include", "ds_topk.h")
LIB = os.path.join(PKG, "libdstopk.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def nvcc_path():
    p = shutil.which("nvcc")
    if p:
        return p
    cand = "/usr/local/cuda/bin/nvcc"
    if os.path.exists(cand):
        return cand
    raise RuntimeError("nvcc not found: cannot build libdstopk.so")


def sources():
    files = [HEADER]
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh", ".h")):
            files.append(os.path.join(CSRC, f))
    return files


def stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in sources())


def build(force=False, verbose=False):
    """Compile csrc/lib.cu into libdstopk.so next to this file; return its path."""
    if not force and not stale():
        return LIB
    tmp = LIB + ".tmp"
    cmd = [nvcc_path()] + NVCC_FLAGS + ["-o", tmp, os.path.join(CSRC, "lib.cu")]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
