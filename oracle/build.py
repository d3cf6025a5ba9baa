"""Compile the CPU oracle (plain C, gcc) into oracle/_oracle.so.

Test infrastructure only.  ``-ffp-contract=off`` keeps gcc from fusing the
oracle's double-precision a*b+c into FMAs, so the code computes what it says;
the one fused multiply-add the oracle wants (the fp32 projection) is an
explicit ``fmaf`` call.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCES = ["haar.c", "fsq.c"]
TARGET = os.path.join(HERE, "_oracle.so")


def build(force: bool = False) -> str:
    srcs = [os.path.join(HERE, s) for s in SOURCES]
    if not force and os.path.exists(TARGET):
        newest = max(os.path.getmtime(s) for s in srcs)
        if os.path.getmtime(TARGET) >= newest:
            return TARGET
    cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-Wall", "-Wextra", "-o", TARGET + ".tmp"] + srcs + ["-lm"]
    subprocess.run(cmd, check=True)
    os.replace(TARGET + ".tmp", TARGET)
    return TARGET


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
