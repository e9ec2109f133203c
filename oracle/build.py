"""Compile the fp64 CPU oracle (test infrastructure) into oracle/libslay_oracle.so.

Plain gcc with OpenMP; no CUDA, no file of the library is read or linked.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libslay_oracle.so")
SRC = os.path.join(HERE, "slay_oracle.c")
HDR = os.path.join(HERE, "slay_oracle.h")


def build(force: bool = False) -> str:
    """Build the oracle library if it is missing or older than its sources."""
    newest = max(os.path.getmtime(SRC), os.path.getmtime(HDR))
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared",
           "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
