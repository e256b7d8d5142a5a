"""Builds the oracle's shared library (plain C) in place: oracle/liborc.so.

Test infrastructure only.  Compiled with -ffp-contract=off so that no f32
product is fused into a sum, and with OpenMP for the row-parallel CPU baseline.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(HERE, "liborc.so")


def build_oracle(verbose: bool = False) -> str:
    src = os.path.join(HERE, "qmv_oracle.c")
    out = library_path()
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, src, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build_oracle(verbose=True))
