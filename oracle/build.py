"""Compiles the fp64 C oracle (``hstu_oracle.c``) into ``oracle/libhstu_oracle.so``.

Test infrastructure: the oracle checks the CUDA library and is never part of it.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "hstu_oracle.c")
LIB = os.path.join(HERE, "libhstu_oracle.so")


def build(force: bool = False) -> str:
    """Builds the shared library if it is missing or older than its source; returns its path."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-Wall", "-Wextra",
           "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
