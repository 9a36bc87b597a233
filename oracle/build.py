"""Compile the fp64 oracle (plain C, OpenMP) into a shared library.

Building the checker is not using it: ``__graft_entry__.build()`` calls this so
the library exists next to its source; only tests, the smoke check and the CPU
baseline load it.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "mea_oracle.c")


def default_library_path() -> str:
    return os.path.join(HERE, "liboracle.so")


def build_oracle(src: str = SOURCE, out: str | None = None, extra_flags=()) -> str:
    """gcc -O2 -fopenmp; portable x86-64 code so the library runs on any host."""
    out = out or default_library_path()
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-ffp-contract=off",
           *extra_flags, src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build_oracle(*sys.argv[1:2]))
