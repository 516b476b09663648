"""Compile the fp64 CPU oracle (``kda_oracle.c``) into ``libkda_oracle.so``.

Test infrastructure: the library is loaded by the test suite, the smoke check
and the benchmark's CPU-baseline leg, never by the CUDA product path.
Run as ``python oracle/build.py`` or call :func:`build`.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kda_oracle.c")
LIB = os.path.join(HERE, "libkda_oracle.so")


def build(force: bool = False) -> str:
    """Build the shared library if it is missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    # -O2 without -ffast-math: the oracle keeps IEEE double semantics and the
    # written operation order (no reassociation, no FMA contraction).
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
           "-std=c11", "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
