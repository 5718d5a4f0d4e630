"""Build the fp64 CPU oracle (``liboracle_far.so``) with gcc.

Test infrastructure only: the library it builds is loaded by the test suite,
the smoke check and the bench's CPU-baseline leg, never by the product path.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "far_oracle.c")
LIB = os.path.join(HERE, "liboracle_far.so")

# Plain ISO C, no fast-math and no contraction into FMA: every double
# operation rounds once, exactly as written in the source.
CFLAGS = ["-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-Wall", "-Wextra"]


def build(src: str = SRC, out: str = LIB, force: bool = False) -> str:
    """Compile ``src`` into the shared library ``out`` (skipped when up to date)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
