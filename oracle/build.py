"""Compile the plain-C oracle into oracle/libmoe_q4_oracle.so with gcc.

Test infrastructure: the oracle is built so that the tests, the smoke check and
the benchmark's CPU baseline can run it; nothing on the product path loads it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_q4_oracle.c")
LIB = os.path.join(HERE, "libmoe_q4_oracle.so")

# -ffp-contract=off: no fused multiply-add contraction, so every binary64 and
# binary32 operation rounds exactly as written in the source.
CFLAGS = ["-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11"]


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", *CFLAGS, SRC, "-o", LIB, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
