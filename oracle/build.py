"""Build the CPU oracle library (oracle/liboracle.so) with gcc.

Test infrastructure: the oracle is compiled with IEEE-exact settings (no fast
math, no FMA contraction) and OpenMP across independent rows and tiles.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fp8bq_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC",
          "-fvisibility=hidden", "-std=c11", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile liboracle.so if it is missing or older than its source; return its path."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    subprocess.run(["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
