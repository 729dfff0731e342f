"""Build the CPU oracle shared library (test infrastructure only).

    python oracle/build.py            # builds oracle/liboracle.so
    python oracle/build.py -DNAME=1   # extra defines (used by the planted-mistake tests)
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fa4_oracle.c")


def build(out: str | None = None, defines: tuple[str, ...] = (), force: bool = False) -> str:
    out = out or os.path.join(HERE, "liboracle.so")
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(SRC):
        return out
    cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", out + ".tmp", SRC, "-lm", *defines]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(defines=tuple(sys.argv[1:]), force=True))
