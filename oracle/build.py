"""Compile the CPU oracle (oracle.c) into oracle/liboracle.so.

Test infrastructure: the oracle is a checker, not part of the product path.
Building it is allowed anywhere; calling it is reserved for the tests, the
smoke check and the benchmark's CPU-baseline leg.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-pthread"]


def build(src: str = SRC, out: str = LIB, extra=()) -> str:
    """Compile src into the shared library out (only when out is stale)."""
    if os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src) and not extra:
        return out
    cmd = ["gcc", *CFLAGS, *extra, "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(*sys.argv[1:2]))
