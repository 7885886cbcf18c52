"""Build the CUDA twin of the workload generator (synth/libloopvq_synth.so), sm_100a."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "synth_gen.cu")
LIB = os.path.join(HERE, "libloopvq_synth.so")


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
                               "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-o", LIB, SRC])
    return LIB


if __name__ == "__main__":
    print(build(force=True))
