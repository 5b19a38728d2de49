"""Compile the fp64 CPU oracle into oracle/liboracle.so (gcc, OpenMP, no fast-math).

TEST INFRASTRUCTURE ONLY: the oracle checks the CUDA library; it is never part
of the product path.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "wkv_oracle.c")
SOURCES = [SRC, os.path.join(HERE, "wkv5_oracle.c")]
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Build liboracle.so if it is missing or older than its source; return its path."""
    if not force and os.path.exists(LIB) and all(os.path.getmtime(LIB) >= os.path.getmtime(p) for p in SOURCES):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", "-Wall", "-Wextra",
           "-o", LIB + ".tmp", *SOURCES, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
