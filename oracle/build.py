"""Builds the oracle's shared library with gcc (plain C, OpenMP).

TEST INFRASTRUCTURE: the oracle is only loaded by the test suite, the
package smoke check and the benchmark's CPU-baseline / reference arm.

    python oracle/build.py            # writes oracle/libattn_oracle.so
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "attn_oracle.c")
LIB = os.path.join(HERE, "libattn_oracle.so")


def build(out=LIB, plant=0, force=False):
    """Compiles attn_oracle.c into `out`; `plant` != 0 builds a planted-mistake variant."""
    if (not force and plant == 0 and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(SRC)):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-Wall", "-Wextra", f"-DORACLE_PLANT={int(plant)}", SRC, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
