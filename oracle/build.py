"""Compile the CPU oracle (dq_oracle.c) into oracle/liboracle.so with gcc.

Test infrastructure: only the test suite, the smoke check and the benchmark's
CPU-baseline leg use the oracle.  Building it is part of ``build()`` so that
the checker exists wherever the library is built.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "dq_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

# -ffp-contract=off: no FMA contraction, each fp32 op rounds on its own.
# -fno-fast-math: IEEE division and rounding, no reciprocal tricks.
# -fwrapv: int32 overflow wraps (the int64 twin would expose it).
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fwrapv",
          "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    cmd = ["gcc", *CFLAGS, "-o", LIB, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
