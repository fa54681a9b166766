"""Compile the fp64 CPU oracle (csa_oracle.c) into liboracle's shared object.

Test infrastructure: the product library never links or loads the result.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csa_oracle.c")
LIB = os.path.join(HERE, "libcsa_oracle.so")


def build(force: bool = False) -> str:
    """Build libcsa_oracle.so next to its source (gcc, -O2, OpenMP)."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fopenmp", "-fPIC", "-shared",
           SRC, "-o", LIB + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
