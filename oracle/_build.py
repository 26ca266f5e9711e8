"""Compile the CPU fp64 oracle (plain C + OpenMP).  Test infrastructure only."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "liboracle.so")


def build(force=False):
    src = os.path.join(HERE, "oracle.c")
    if force or not os.path.exists(SO) or os.path.getmtime(src) > os.path.getmtime(SO):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-o", SO, src, "-lm"])


if __name__ == "__main__":
    build(force=True)
