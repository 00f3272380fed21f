"""Build synth/libkvsynth.so (the GPU twin of the seeded generator) for sm_100a."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "synth_gen.cu")
LIB = os.path.join(HERE, "libkvsynth.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def build(verbose: bool = False) -> str:
    hdr = os.path.join(ROOT, "include", "kvsynth.h")
    newest = max(os.path.getmtime(SRC), os.path.getmtime(hdr))
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < newest:
        # -fmad=false: every fp64 operation is rounded on its own, as in the numpy twin
        cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
               "-fmad=false", "-Xcompiler", "-fPIC", "-I" + os.path.join(ROOT, "include"), "-shared", SRC,
               "-o", LIB]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed:\n{r.stdout}\n{r.stderr}")
    if verbose:
        print(LIB)
    return LIB


if __name__ == "__main__":
    build(verbose=True)
