"""Compile the CPU oracle (test infrastructure only) into oracle/liblaoracle.so.

Plain gcc, -O3, OpenMP over (request, head) tiles.  No -march=native: the shared
object may be built on one host and loaded on another.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "la_oracle.c")
LIB = os.path.join(HERE, "liblaoracle.so")


def build(force: bool = False) -> str:
    deps = [SRC, os.path.join(HERE, "la_oracle.h")]
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(p) for p in deps)):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-std=c11", "-O3", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
