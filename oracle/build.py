"""Compile the CPU oracle (plain C) into oracle/liboracle.so.

Test infrastructure: the oracle is built alongside the CUDA library so that
the test-suite and the benchmark's CPU-baseline leg can load it; building it
does not put it on the product path.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
OUT = os.path.join(HERE, "liboracle.so")

FLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fexcess-precision=standard",
         "-fopenmp", "-shared", "-fPIC", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    if not force and os.path.exists(OUT) and os.path.getmtime(OUT) >= os.path.getmtime(SRC):
        return OUT
    cmd = ["gcc", *FLAGS, SRC, "-o", OUT + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
