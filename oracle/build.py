"""Build the CPU oracle shared library (test infrastructure only).

    python -m oracle.build

Compiles tf4_oracle.c with gcc, -O2 -ffp-contract=off (every float
expression is exactly one IEEE operation), into oracle/libtf4_oracle.so.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "tf4_oracle.c")
LIB = os.path.join(HERE, "libtf4_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= max(
        os.path.getmtime(SRC), os.path.getmtime(os.path.join(HERE, "tf4_oracle.h"))
    ):
        return LIB
    cmd = [
        "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wextra",
        "-fPIC", "-shared", "-o", LIB + ".tmp", SRC, "-lm",
    ]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
