"""Compile the C oracle into ``oracle/_sinkhorn_oracle.so`` (gcc, OpenMP, -O3).

The hot loops carry gcc ``target_clones`` (avx512f / avx2 / baseline), so one
build runs on any x86-64 host.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "sinkhorn_oracle.c")
LIB = os.path.join(HERE, "_sinkhorn_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-Wall", "-std=c11", SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
