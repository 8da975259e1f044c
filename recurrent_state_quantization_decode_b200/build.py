"""Build libleapquant.so in-tree with nvcc for sm_100a (B200).

    python -m recurrent_state_quantization_decode_b200.build [--force] [--verbose]

The CUDA runtime is linked statically, so the library loads without a GPU and
works next to the runtime PyTorch ships.  --verbose passes -Xptxas -v.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libleapquant.so")
SOURCES = [os.path.join(CSRC, f) for f in ("lq_decode.cu", "lq_fp32.cu", "lq_checkpoint.cu",
                                            "lq_hostio.cu", "lq_capi.cu", "lq_noalloc.cu")]
DEPS = SOURCES + [os.path.join(CSRC, h) for h in ("lq_internal.h", "lq_checkpoint.h",
                                                          "lq_hostio.h", "lq_capi_internal.h")] + \
    [os.path.join(INCLUDE, "leapquant.h")]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libleapquant.so")
    return path


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    cmd = [nvcc(), "-O3", "-lineinfo", "-std=c++17",
           "-gencode", "arch=compute_100a,code=sm_100a",
           "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
           "-I", INCLUDE, *SOURCES, "-o", LIB + ".tmp"]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
