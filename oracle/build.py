"""Build the CPU oracle shared library (``liborc_fp8.so``) with gcc.

The oracle is test infrastructure: this builder only compiles it, so that
the tests and the bench's CPU-baseline leg can load it.  Flags keep IEEE
single-precision semantics: no fast-math, no FMA contraction.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "liborc_fp8.so")
SRC = os.path.join(HERE, "fp8_oracle.c")
HDR = os.path.join(HERE, "fp8_oracle.h")

CFLAGS = ["-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
          "-fPIC", "-shared", "-fopenmp", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile the oracle if its source is newer than the library."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(SRC), os.path.getmtime(HDR))):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    subprocess.run(["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
