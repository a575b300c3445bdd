"""Compile the fp64 CPU oracle (test infrastructure) into oracle/libjloracle.so.

Plain gcc, -O2, OpenMP, IEEE semantics (no fast-math, no -march=native so the
built library runs on any x86-64 host it is copied to).
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "jl_oracle.c")
LIB = os.path.join(HERE, "libjloracle.so")


def build(src: str = SRC, out: str = LIB, force: bool = False) -> str:
    """Build the oracle shared library if it is missing or older than its source."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-Wno-unused-parameter", src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force=True))
