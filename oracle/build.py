"""Builds the CPU oracle (test infrastructure only) into ``oracle/liborc.so``."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liborc.so")


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(SRC) > os.path.getmtime(LIB):
        # no -ffast-math: the oracle keeps IEEE fp64 semantics and plain summation order
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", LIB, SRC, "-lm"])
    return LIB


if __name__ == "__main__":
    build(force=True)
