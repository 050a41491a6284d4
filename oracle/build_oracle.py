"""Build the CPU oracle library (``oracle/liblqq_oracle.so``) with gcc.

Test infrastructure: the oracle checks the CUDA library and is never part of
its path.  Plain ``-O2`` without fast-math and without FP contraction, so
every fp32 division and rounding is the IEEE operation the source names.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lqq_oracle.c")
LIB = os.path.join(HERE, "liblqq_oracle.so")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wextra", "-shared", "-fPIC",
           "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
