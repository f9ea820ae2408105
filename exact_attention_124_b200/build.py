"""Build the sm_100a CUDA library in-tree (``libattn_b200.so`` next to this file).

    python -m exact_attention_124_b200.build [--force] [-v]

nvcc cross-compiles for B200 (``-gencode arch=compute_100a,code=sm_100a``)
without a GPU present.  The library is one translation unit
(``csrc/attn_lib.cu``) exposing the C ABI declared in ``include/``.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SO = os.path.join(HERE, "libattn_b200.so")
SRC = os.path.join(HERE, "csrc", "attn_lib.cu")
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared"]


def _inputs():
    return (glob.glob(os.path.join(HERE, "csrc", "*")) +
            glob.glob(os.path.join(ROOT, "include", "*.h")))


def needs_build() -> bool:
    if not os.path.exists(SO):
        return True
    t = os.path.getmtime(SO)
    return any(os.path.getmtime(f) > t for f in _inputs())


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if a source is newer than it (or ``force``)."""
    if not force and not needs_build():
        return SO
    tmp = SO + ".tmp"
    cmd = [nvcc(), *NVCC_FLAGS, "-I" + os.path.join(ROOT, "include"), "-o", tmp, SRC]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, SO)
    return SO


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(SO)
