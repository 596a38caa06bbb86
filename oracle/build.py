"""Compile the CPU oracle (zo_oracle.c) into oracle/liboracle.so with gcc.

Test infrastructure: the library this builds is loaded only by the tests, the smoke
check and the benchmark's CPU-baseline leg.  -ffp-contract=off keeps every fp32/fp64
operation a separate IEEE operation, as the oracle's fixed summation orders assume.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "zo_oracle.c")
OUT = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(OUT) and os.path.getmtime(OUT) >= os.path.getmtime(SRC):
        return OUT
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wextra", "-o", OUT + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
