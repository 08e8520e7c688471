"""Compile the fp64 CPU oracle (oracle.c) into oracle/liboracle.so with gcc.

Test infrastructure: the oracle is only loaded by the tests, the smoke check and
the benchmark's CPU-baseline leg.  Building it is not using it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def compile_c(src: str, out: str, extra=()) -> None:
    """gcc one oracle source into a shared library at `out` (written atomically);
    `extra` flags come last (e.g. -w for deliberately altered copies)."""
    cmd = [
        "gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
        "-fPIC", "-shared", "-Wall", "-Wextra", "-Wno-unused-parameter", *extra,
        src, "-o", out + ".tmp", "-lm",
    ]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    compile_c(SRC, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
