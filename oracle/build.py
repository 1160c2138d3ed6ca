"""Build the fp64 CPU oracle shared library (test infrastructure only).

    python oracle/build.py

Compiles ``pararnn_oracle.c`` with gcc into ``_liboracle.so`` beside it.
No fast-math: the oracle's operations are plain IEEE double operations.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pararnn_oracle.c")
OUT = os.path.join(HERE, "_liboracle.so")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(OUT)
            and os.path.getmtime(OUT) >= os.path.getmtime(SRC)):
        return OUT
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
           "-fno-fast-math", "-ffp-contract=off", "-o", OUT, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
