"""Compile the CPU oracle (plain C, OpenMP) into ``oracle/libkvq_oracle.so``.

Contraction of multiplies and adds into FMA is switched off: the quantizers
are defined as separately rounded fp32 operations.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(HERE, "libkvq_oracle.so")


def build_oracle(verbose: bool = False) -> str:
    src = os.path.join(HERE, "kvq_oracle.c")
    out = library_path()
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-Wall", "-o", tmp, src, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build_oracle(verbose=True))
