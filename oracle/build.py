"""Compile the C oracle into oracle/liboracle.so (gcc, OpenMP, no fast-math).

Test infrastructure: building the checker is not using it on the product path.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


FLAGS = ["-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra"]


def compile_source(src: str, out: str, quiet: bool = False) -> None:
    """gcc ``src`` into the shared library ``out`` with the oracle's flags."""
    subprocess.run(["gcc", *FLAGS, "-o", out, src, "-lm"], check=True,
                   capture_output=quiet)


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    compile_source(SRC, tmp)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
