"""Compile the oracle's C part (assign.c) into oracle/liboracle.so with gcc.

    python -m oracle.build_oracle

Flags: -O2 -ffp-contract=off (no fused multiply-add, no reassociation, so each
sum is the plain left-to-right float64 sum written in the source) and OpenMP
over rows.  Test infrastructure only.
"""
from __future__ import annotations

import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "assign.c")
LIB = os.path.join(HERE, "liboracle.so")


def build() -> str:
    if os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        raise RuntimeError("no C compiler for the oracle")
    tmp = LIB + f".{os.getpid()}.tmp"
    cmd = [cc, "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC", SRC, "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"oracle build failed:\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build())
