"""Compile the fp64 CPU oracle (plain C + POSIX threads) into oracle/_attention_ref.so.

Test infrastructure only: the oracle checks the CUDA library and is never on
its path.  No fast-math and no FMA contraction, so every product and sum is
rounded exactly as written in attention_ref.c.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "attention_ref.c")
LIB = os.path.join(HERE, "_attention_ref.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cc = "gcc"
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [cc, "-O2", "-fPIC", "-shared", "-std=c11", "-pthread", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
