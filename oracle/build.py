"""Compile the CPU oracle (plain C, single-threaded) into oracle/libck_oracle.so.

Test infrastructure: the oracle is built so the tests and the benchmark's CPU
baseline can check the CUDA library against it; the product path never loads it.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ck_oracle.c")
HDR = os.path.join(HERE, "ck_oracle.h")
LIB = os.path.join(HERE, "libck_oracle.so")

# -ffp-contract=off: no fused multiply-add, so each fp32 step is one IEEE operation.
CFLAGS = ["-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-Wall", "-Wextra", "-Wno-unused-parameter"]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in (SRC, HDR, __file__))


def build(force: bool = False) -> str:
    if force or needs_build():
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
