"""Build libfa.so in-tree with nvcc for sm_100a.

    python -m exact_tiled_attention_36_b200.build

Compiles csrc/fa_api.cu (which includes the kernel headers) and
csrc/fa_noalloc.cu into exact_tiled_attention_36_b200/libfa.so, with the CUDA runtime linked
statically so the library loads on a machine without a GPU driver (the
driver is reached at run time through the runtime's entry-point query).
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRCS = [os.path.join(HERE, "csrc", "fa_api.cu"), os.path.join(HERE, "csrc", "fa_noalloc.cu")]
DEPS = [os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc"))] + \
       [os.path.join(ROOT, "include", "fa.h")]
LIB = os.path.join(HERE, "libfa.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-std=c++17", "-O3", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC,-O2", "-shared", "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    newest = max(os.path.getmtime(p) for p in DEPS)
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest and not extra:
        return LIB
    tmp = LIB + f".{os.getpid()}.tmp"
    cmd = [NVCC, *FLAGS, *(extra or []), "-I", os.path.join(ROOT, "include"), "-I", os.path.join(HERE, "csrc"),
           *SRCS, "-o", tmp]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
