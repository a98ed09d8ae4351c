"""Build the CPU oracle library (oracle/liborc.so) with gcc.

Test infrastructure only.  Plain C99, -O2, no fast-math and no FMA
contraction, so every fp64 operation rounds exactly as written.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pkv_oracle.c")
HDR = os.path.join(HERE, "pkv_oracle.h")
LIB = os.path.join(HERE, "liborc.so")


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return t < os.path.getmtime(SRC) or t < os.path.getmtime(HDR)


def build(force: bool = False) -> str:
    if force or needs_build():
        cmd = ["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-Wextra", "-o", LIB, SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
