"""Compile the oracle (test infrastructure) into oracle/liboracle.so with gcc.

No fused multiply-add contraction, no fast-math, no vector ISA beyond the
x86-64 baseline: every FP32 operation in the oracle is one IEEE rounding, and
the only fused multiply-add is the explicit fmaf() call.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRCS = [os.path.join(HERE, f) for f in ("damp_oracle.c", "calib_oracle.c")]
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-Wall", "-Wextra", "-Werror"]


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and \
            all(os.path.getmtime(LIB) >= os.path.getmtime(s) for s in SRCS):
        return LIB
    cmd = ["gcc", *CFLAGS, "-o", LIB, *SRCS, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
