"""Builds the CPU oracle (test infrastructure) as a shared library with gcc.

The oracle is compiled without -ffast-math and with -ffp-contract=off, so every FP32
operation in it is one IEEE-754 round-to-nearest-even operation (x86-64 uses SSE2 scalar
arithmetic, never x87 extended precision).
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "nvfp4_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
           "-fno-fast-math", "-fno-unsafe-math-optimizations", "-o", LIB, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
