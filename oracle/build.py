"""Compile the C oracle into ``oracle/liboracle.so`` with gcc.

Test infrastructure: the library is used by tests/, the smoke check and the
benchmark's CPU-baseline leg only.  Plain IEEE double arithmetic: no fast
math, no floating-point contraction.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "spec_verify_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    # A prebuilt library named by SV_ORACLE_LIB takes the place of this one:
    # the mutation test uses it to run the pins against altered copies.
    alt = os.environ.get("SV_ORACLE_LIB")
    if alt:
        return alt
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))
