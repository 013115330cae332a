"""Compile the C oracle (inference and encoding) into oracle/liboracle.so with gcc.

Test infrastructure: the CUDA library never links this.  Flags: -O2 with
OpenMP, no fast-math and no FMA contraction (-ffp-contract=off), so every
floating-point step rounds as written in aqlm_oracle.c.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRCS = [os.path.join(HERE, "aqlm_oracle.c"), os.path.join(HERE, "aqlm_encode_oracle.c")]
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and all(os.path.getmtime(LIB) >= os.path.getmtime(p) for p in SRCS):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", "-o", tmp, *SRCS, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
