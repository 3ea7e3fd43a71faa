"""Build the fp64 CPU oracle (test infrastructure) into oracle/liboracle_qknr.so.

Plain gcc, -O2, no -ffast-math (so libm's pow/sin/cos and the IEEE double
arithmetic stay as written), OpenMP over tokens.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "qknr_oracle.c")
LIB = os.path.join(HERE, "liboracle_qknr.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-Wall", "-Wextra",
           "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
