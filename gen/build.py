"""Builds gen/libmoegen.so (host C half + device CUDA half of the input generator)."""
from __future__ import annotations

import os
import subprocess
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libmoegen.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def build(verbose: bool = False) -> str:
    with tempfile.TemporaryDirectory() as td:
        host_o = os.path.join(td, "gen_host.o")
        dev_o = os.path.join(td, "gen_dev.o")
        cmds = [
            ["gcc", "-O2", "-fPIC", "-ffp-contract=off", "-std=c11", "-I", SRC, "-c",
             os.path.join(SRC, "gen_host.c"), "-o", host_o],
            [NVCC, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
             "--fmad=false", "-Xcompiler", "-fPIC", "-I", SRC, "-c", os.path.join(SRC, "gen_dev.cu"), "-o", dev_o],
            [NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-Xcompiler", "-fPIC", host_o, dev_o, "-o", OUT + ".tmp", "-lpthread", "-lm"],
        ]
        for c in cmds:
            if verbose:
                print(" ".join(c))
            subprocess.run(c, check=True)
        os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(verbose=True))
