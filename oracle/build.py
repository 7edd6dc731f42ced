"""Compiles ``oracle.cpp`` into ``liboracle.so`` beside it (test infrastructure)."""

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")
CMD = ["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread", SRC, "-o", LIB]


def build(force: bool = False) -> str:
    """Builds the oracle library if it is missing or older than its source."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.run(CMD, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
