"""Build the CPU oracle shared library (test infrastructure only).

    python oracle/build.py

Compiles nvfp4_oracle.c with gcc into oracle/liboracle.so.  The flags keep
every fp32 operation a single IEEE round-to-nearest-even operation:
no -ffast-math, no FMA contraction, no reassociation.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "nvfp4_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = [
    "-O2", "-std=c11", "-fPIC", "-shared",
    "-ffp-contract=off", "-fno-fast-math", "-fexcess-precision=standard",
    "-fopenmp",
]


def build(force: bool = False) -> str:
    """Compile the oracle if the .so is missing or older than its source."""
    hdr = os.path.join(HERE, "nvfp4_oracle.h")
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(SRC), os.path.getmtime(hdr))):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
