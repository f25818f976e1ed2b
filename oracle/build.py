"""Compile the CPU oracle (test infrastructure) into ``oracle/liboracle.so``.

Plain gcc, ``-ffp-contract=off`` and no fast-math so that every fp32 step of
the oracle is one IEEE round-to-nearest operation.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pariskv_oracle.c")
HDR = os.path.join(HERE, "pariskv_oracle.h")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    stale = (not os.path.exists(LIB)) or any(
        os.path.getmtime(p) > os.path.getmtime(LIB) for p in (SRC, HDR, __file__))
    if force or stale:
        tmp = LIB + ".%d.tmp" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
