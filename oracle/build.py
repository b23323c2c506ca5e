"""Build script for the CPU oracle (test infrastructure only).

Compiles ``dg_oracle.c`` into ``liboracle.so`` beside this file with gcc,
OpenMP, and strict IEEE semantics (no FMA contraction, no fast-math), so the
quantiser's float divisions and the FP64 sums happen exactly as written.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "dg_oracle.c")
OUT = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(OUT) and os.path.getmtime(OUT) >= max(
            os.path.getmtime(SRC), os.path.getmtime(os.path.join(HERE, "dg_oracle.h"))):
        return OUT
    cmd = ["gcc", "-O2", "-march=x86-64-v2", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-Wall", "-Wextra",
           SRC, "-o", OUT + ".tmp", "-lm"]
    subprocess.check_call(cmd)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
