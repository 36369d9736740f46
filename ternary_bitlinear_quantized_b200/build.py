"""Build libbitnet_b200.so in-tree with nvcc for sm_100a (B200).

Usage: ``python -m ternary_bitlinear_quantized_b200.build [--verbose]``.  nvcc
cross-compiles without a GPU.  The library links the CUDA runtime statically, so it
does not depend on the runtime version torch ships.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libbitnet_b200.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cu", ".cuh"))]


def build(verbose: bool = False, force: bool = False) -> str:
    srcs = sources()
    hdr = os.path.join(os.path.dirname(HERE), "include", "bitnet_b200.h")
    newest = max(os.path.getmtime(p) for p in srcs + [hdr, __file__])
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    cmd = [nvcc(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "--fmad=false", "-Xcompiler", "-fPIC", "-shared",
           "-cudart", "static", "-I", os.path.join(os.path.dirname(HERE), "include"),
           "-o", LIB + ".tmp", os.path.join(CSRC, "bitnet_b200.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose:
        print(res.stderr, file=sys.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force=True)
    print(LIB)
