"""Compile the fp64 CPU oracle into oracle/liboracle.so (test infrastructure).

gcc, -O2 with -ffp-contract=off (no fused multiply-add: every product and sum
rounds on its own, as the oracle's comments state) and OpenMP over images.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "liboracle.so")
SRC = os.path.join(HERE, "oracle.c")


def build(force: bool = False) -> str:
    deps = [SRC, os.path.join(HERE, "oracle.h")]
    if not force and os.path.exists(SO) and all(
            os.path.getmtime(SO) >= os.path.getmtime(d) for d in deps):
        return SO
    tmp = SO + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-Wall", "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, SO)
    return SO


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
