"""Compile the fp64 CPU oracle (oracle.c) into oracle/liboracle.so with gcc.

Test infrastructure only: the oracle is built so that the tests, the smoke check and the
CPU-baseline leg of the benchmark can call it.  No optimisation flags that change fp64
semantics are used (no -ffast-math, no FMA contraction).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
HDR = os.path.join(HERE, "oracle.h")
LIB = os.path.join(HERE, "liboracle.so")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    lib_t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > lib_t for p in (SRC, HDR, __file__))


def build(force: bool = False) -> str:
    if force or needs_build():
        cmd = ["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-ffp-contract=off", "-fPIC",
               "-shared", "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
