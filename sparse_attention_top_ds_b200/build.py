"""Build libdstopk.so in-tree for sm_100a with nvcc (no JIT cache), and next
to it libdstopk_debug.so, the same library compiled with DS_DEBUG (device range
checks that record DS_ERR_RANGE in the status word).

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
LIB_DEBUG = os.path.join(PKG, "libdstopk_debug.so")

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


def stale(lib=LIB):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in sources())


def build(force=False, verbose=False):
    """Compile csrc/lib.cu into libdstopk.so and libdstopk_debug.so next to
    this file (the two nvcc runs side by side); return the release path."""
    jobs = []
    for lib, extra in ((LIB, []), (LIB_DEBUG, ["-DDS_DEBUG"])):
        if not force and not stale(lib):
            continue
        tmp = lib + ".tmp"
        cmd = [nvcc_path()] + NVCC_FLAGS + extra + ["-o", tmp, os.path.join(CSRC, "lib.cu")]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
        jobs.append((lib, tmp, proc))
    errors = []
    for lib, tmp, proc in jobs:
        out, err = proc.communicate()
        if proc.returncode != 0:
            errors.append(f"nvcc failed for {os.path.basename(lib)}:\n" + out + err)
        else:
            os.replace(tmp, lib)
    if errors:
        raise RuntimeError("\n".join(errors))
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
