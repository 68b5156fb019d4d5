"""Build step for the fp64 CPU oracle (test infrastructure).

Compiles ``ss_oracle.c`` (forward) and ``ss_oracle_bwd.c`` (gradients) with
gcc into ``liboracle.so`` beside them.  Strict
IEEE arithmetic: no -ffast-math, no contraction of a*b+c into an FMA, so the
oracle rounds exactly as its C source reads.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ss_oracle.c")
SRCS = [SRC, os.path.join(HERE, "ss_oracle_bwd.c")]
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= max(map(os.path.getmtime, SRCS)):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
           *SRCS, "-o", LIB + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
