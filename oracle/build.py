"""Compile the C oracle into ``oracle/liboracle.so`` (test infrastructure only).

Plain gcc, no fast-math, so every double operation is an IEEE-754 binary64
operation with round-to-nearest-even, as the oracle's readings assume.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
          "-Wall", "-Wextra"]


def build(src: str = SRC, out: str = LIB, strict: bool = True) -> str:
    """Compile ``src`` into the shared library ``out`` and return its path.
    ``strict`` turns warnings into errors (off only for deliberately broken
    copies made by the mutation tests)."""
    cmd = ["gcc", *CFLAGS, *(["-Werror"] if strict else []), "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def ensure_built() -> str:
    """Build the oracle library if it is missing or older than its source."""
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        build()
    return LIB


if __name__ == "__main__":
    print(build(*sys.argv[1:2]))
