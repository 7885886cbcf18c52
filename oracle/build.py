"""Compile the CPU checker library (test infrastructure; never linked into the CUDA library)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "loopvq_oracle.c")
LIB = os.path.join(HERE, "libloopvq_oracle.so")


def build(force: bool = False) -> str:
    """Build with strict IEEE semantics: no fast-math, no FMA contraction."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", LIB, SRC, "-lm"])
    return LIB


if __name__ == "__main__":
    print(build(force=True))
