"""Build the CPU oracle shared library (test infrastructure only).

    python oracle/build_oracle.py

Compiles ``nf4_oracle.c`` with gcc into ``oracle/liboracle_nf4.so``.  No
contraction of multiply-adds and no fast-math, so that every fp32 / fp64 step
in the C source is one IEEE operation rounded to nearest even.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "nf4_oracle.c")
OUT = os.path.join(HERE, "liboracle_nf4.so")
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fexcess-precision=standard",
          "-Wall", "-Wextra", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    if not force and os.path.exists(OUT) and os.path.getmtime(OUT) >= max(
            os.path.getmtime(SRC), os.path.getmtime(os.path.join(HERE, "nf4_oracle.h"))):
        return OUT
    tmp = OUT + ".tmp.%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
