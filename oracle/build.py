"""Build the CPU oracle shared library (test infrastructure: only tests, the smoke check and the
benchmark's CPU-baseline leg load it).

    python oracle/build.py          # writes oracle/libs3r_oracle.so
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "s3r_oracle.c")
LIB = os.path.join(HERE, "libs3r_oracle.so")


def build(force: bool = False) -> str:
    """Compile s3r_oracle.c with gcc (-O2, no fast-math: IEEE double arithmetic as written)."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= max(
        os.path.getmtime(SRC), os.path.getmtime(os.path.join(HERE, "s3r_oracle.h"))
    ):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared", "-pthread",
           "-Wall", "-Wextra", "-o", LIB, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
