"""Compile the oracle's C source into oracle/liblora_oracle.so (gcc, -O2, no
fast-math, OpenMP over independent tokens).

Test infrastructure: the oracle is a checker, never part of the product path.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lora_oracle.c")
LIB = os.path.join(HERE, "liblora_oracle.so")


def build(force: bool = False, src: str = SRC, out: str = LIB) -> str:
    """Build the shared library if it is missing or older than its source."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-fPIC", "-shared", "-std=c99", "-Wall", "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
