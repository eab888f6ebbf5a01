"""Compile the C oracle into a shared library (plain gcc, -O2, no fast-math).

Test infrastructure: see ``oracle/__init__.py``.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bdscan_oracle.c")


def lib_path(mutant: int = 0) -> str:
    return os.path.join(HERE, "liboracle.so" if mutant == 0 else f"liboracle_m{mutant}.so")


def build(mutant: int = 0, force: bool = False) -> str:
    out = lib_path(mutant)
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(SRC)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-Wextra",
           f"-DORACLE_MUTANT={int(mutant)}", "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force=True))
