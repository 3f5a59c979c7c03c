"""Compile the CPU oracle (oracle.c) into oracle/liboracle.so.

Test infrastructure: the oracle is built here so that the tests, the smoke
check and the benchmark's CPU-baseline leg can load it; the product library
never links it.  Flags: -O2 with contraction of multiply-adds disabled, so
every floating-point operation is the one written in the source.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
OUT = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(OUT) and os.path.getmtime(OUT) >= max(
        os.path.getmtime(SRC), os.path.getmtime(os.path.join(HERE, "oracle.h"))
    ):
        return OUT
    tmp = OUT + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
