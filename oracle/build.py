"""Compile the C oracle (test infrastructure) into ``oracle/libcq_oracle.so``.

The oracle is built with IEEE-faithful flags: no fast-math and no floating-point
contraction, so every binary32 operation in ``cq_oracle.c`` is rounded on its own.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cq_oracle.c")
LIB = os.path.join(HERE, "libcq_oracle.so")

CFLAGS = ["-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp"
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, SRC, "-lpthread", "-lm"])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
