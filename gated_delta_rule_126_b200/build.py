"""Build the KDA CUDA library in-tree: ``gated_delta_rule_126_b200/lib/libkda_b200.so``.

Every kernel is compiled for sm_100a only (``-gencode arch=compute_100a,code=sm_100a``);
the CUDA runtime is linked statically, so the library needs only the driver.
Run ``python -m gated_delta_rule_126_b200.build`` (nvcc cross-compiles without a GPU).
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(PKG, "lib")
LIB_PATH = os.path.join(LIB_DIR, "libkda_b200.so")
SOURCES = ["kda_api.cu", "kda_decode.cu", "kda_prefill_simt.cu", "kda_prefill_tc.cu", "kda_noalloc.cu",
           "kda_epilogue.cu", "kda_prologue.cu", "kda_split.cu", "kda_selftest.cu",
           "kda_backward.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def _stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "kda.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every source and link the shared library; return its path."""
    if not force and not _stale():
        return LIB_PATH
    os.makedirs(os.path.join(PKG, "_build"), exist_ok=True)
    os.makedirs(LIB_DIR, exist_ok=True)
    objs = []
    for src in SOURCES:
        obj = os.path.join(PKG, "_build", src.replace(".cu", ".o"))
        cmd = [NVCC, *ARCH, *FLAGS, "-I", INCLUDE, "-I", CSRC, "-c",
               os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = LIB_PATH + ".tmp"
    cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-lcuda"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
