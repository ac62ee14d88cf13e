"""Builds the CPU oracle's shared library (oracle/liboracle.so) with gcc.

Test infrastructure only: the product library never links or loads it.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lbq_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

# Strict IEEE: no fused multiply-add contraction, no fast-math reassociation.
CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
          "-Wall", "-Wextra", "-shared", "-fPIC", "-std=c11"]


def build_oracle(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build_oracle(force=True))
