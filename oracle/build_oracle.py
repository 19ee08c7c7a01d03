"""Compile the fp64 CPU oracle (test infrastructure only) into a shared object.

The oracle is plain C with OpenMP; gcc builds it in a second.  The product
library never links it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moba_oracle.c")
LIB = os.path.join(HERE, "_moba_oracle.so")


def build(force: bool = False) -> str:
    """Build oracle/_moba_oracle.so if missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-Wall", "-Wextra", "-o", tmp, SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
