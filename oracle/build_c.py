"""Compiles the oracle's C weight generator (oracle/csrc/weightgen.c) with gcc."""

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "weightgen.c")
LIB = os.path.join(HERE, "libweightgen.so")


def build() -> str:
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.run(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC", SRC,
                        "-o", LIB], check=True)
    return LIB


if __name__ == "__main__":
    print(build())
