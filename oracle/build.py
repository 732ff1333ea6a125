"""Builds the fp64 C++ oracle, oracle/libmoe_oracle.so (plain g++, no CUDA)."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.cpp")
OUT = os.path.join(HERE, "libmoe_oracle.so")

# -ffp-contract=off: every a * b + c is a rounded product then a rounded sum,
# as written (no fused multiply-add).
FLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", "-ffp-contract=off"]


def up_to_date() -> bool:
    return os.path.exists(OUT) and os.path.getmtime(OUT) >= max(os.path.getmtime(SRC), os.path.getmtime(__file__))


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return OUT
    cmd = ["g++", *FLAGS, SRC, "-o", OUT + ".tmp"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    import sys

    print(build(force="--force" in sys.argv, verbose=True))
